// Permute: histogram of the T*k slots per expert, inclusive scan (bins), a
// stable counting sort by expert id on the low max(ceil(log2 E),1) key bits,
// and capacity drop by arrival order, in one kernel with no host sync.
//
// Sources: "MegaBlocks 01 - why MoE is hard", section 4.1 (sort the flat top-k
// expert ids, histogram, inclusive cumsum = bins; cub radix sort given an
// end_bit so only the low key bits are sorted; histogram and sort were two
// kernels there), sections 3 and 4.2 (capacity), 4.4-4.5 (an expert keeps its
// first C slots in sorted order; the rest are dropped silently).
//
// One CTA of 1024 threads walks the slots in chunks of 1024, in slot order.
// Inside a chunk, __match_any_sync groups the lanes of a warp that carry the
// same key; a lane's rank inside its warp is the popcount of the lower peers;
// the per-warp counts are scanned across the 32 warps per key, on top of a
// running per-key total. That yields each slot's rank among the earlier slots
// of its expert (the stable order) in a single pass. The counting sort with
// 2^bits buckets is then one scatter: position = start[e] + rank.
// The single CTA keeps the order exact without cross-block waits; S <= 65536
// slots at the workloads here, a few microseconds.
#include "common.cuh"
#include <algorithm>
#include <climits>

namespace moe {

namespace {

constexpr int kThreads = 1024;
constexpr int kMaxE = 256;

__global__ void __launch_bounds__(kThreads)
permute_kernel(const int32_t* __restrict__ idx, int S, int E, unsigned key_mask, long long cap,
               int binned, int32_t* __restrict__ counts, int32_t* __restrict__ bins,
               int32_t* __restrict__ sorted_slot, int32_t* __restrict__ slot_to_row,
               int32_t* __restrict__ row_slot, uint8_t* __restrict__ drop,
               int32_t* __restrict__ kept, int32_t* __restrict__ seg, int32_t* __restrict__ rank_g,
               Control* ctl, AuxJob job, int has_job) {
  pdl_begin();
  __shared__ __align__(16) int hist[32][kMaxE + 1];
  __shared__ int running[kMaxE];
  __shared__ int start_s[kMaxE];
  __shared__ int seg_s[kMaxE + 1];
  __shared__ int kept_s[kMaxE];
  __shared__ int wtot_c[8], wtot_k[8];
  __shared__ int maxc_s;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const unsigned lt_mask = (1u << lane) - 1u;

  for (int i = tid; i < 32 * (kMaxE + 1); i += kThreads) (&hist[0][0])[i] = 0;
  for (int i = tid; i < kMaxE; i += kThreads) running[i] = 0;
  if (tid == 0) maxc_s = 0;
  __syncthreads();

  // ---- pass 1: stable rank of every slot within its expert
  int e_next = tid < S ? __ldg(idx + tid) : -1;  // prefetched one chunk ahead
  for (int base = 0; base < S; base += kThreads) {
    const int s = base + tid;
    int e = e_next;
    e_next = (s + kThreads < S) ? __ldg(idx + s + kThreads) : -1;
    if (s < S) {
      if (e < 0 || e >= E) {
        set_error(ctl, MOE_DEVERR_EXPERT_RANGE);
        e = -1;
      }
    }
    const unsigned key = e >= 0 ? (static_cast<unsigned>(e) & key_mask) : 0xffffffffu;
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    const int r_in_warp = __popc(peers & lt_mask);
    if (e >= 0 && lane == __ffs(peers) - 1) hist[warp][key] = __popc(peers);
    __syncthreads();
    // exclusive scan over the 32 warps, one key per warp at a time; lane = warp index
    for (int ke = warp; ke < E; ke += 32) {
      const int c = hist[lane][ke];
      int incl = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += n;
      }
      const int run = running[ke];
      __syncwarp();
      hist[lane][ke] = run + incl - c;
      if (lane == 31) running[ke] = run + incl;
    }
    __syncthreads();
    if (e >= 0) rank_g[s] = hist[warp][key] + r_in_warp;
    __syncthreads();
    for (int i = tid; i < 32 * E; i += kThreads) hist[i / E][i % E] = 0;
    __syncthreads();
  }

  // ---- counts, bins (inclusive), kept = min(count, C), seg (exclusive) over E <= 256
  // Binned layout: bin size C = cap, or the largest count when cap is none.
  if (binned && cap == LLONG_MAX && tid < E) atomicMax(&maxc_s, running[tid]);
  __syncthreads();
  const long long bin = binned ? (cap == LLONG_MAX ? static_cast<long long>(maxc_s) : cap) : 0;
  int c = 0, kp = 0, ci = 0, ki = 0;
  if (tid < 256) {
    c = tid < E ? running[tid] : 0;
    const long long lim = binned ? bin : cap;
    kp = static_cast<int>(c < lim ? c : lim);
    ci = c;
    ki = kp;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int n1 = __shfl_up_sync(0xffffffffu, ci, off);
      const int n2 = __shfl_up_sync(0xffffffffu, ki, off);
      if (lane >= off) { ci += n1; ki += n2; }
    }
    if (lane == 31) { wtot_c[warp] = ci; wtot_k[warp] = ki; }
  }
  __syncthreads();
  if (tid < 256) {
    int pc = 0, pk = 0;
    for (int w = 0; w < warp; ++w) { pc += wtot_c[w]; pk += wtot_k[w]; }
    ci += pc;
    ki += pk;
    if (tid < E) {
      const int sg = binned ? static_cast<int>(tid * bin) : ki - kp;
      counts[tid] = c;
      bins[tid] = ci;
      kept[tid] = kp;
      seg[tid] = sg;
      start_s[tid] = ci - c;
      seg_s[tid] = sg;
      kept_s[tid] = kp;
    }
    if (tid == E - 1) {
      const int end = binned ? static_cast<int>(E * bin) : ki;
      seg[E] = end;
      seg_s[E] = end;
    }
  }
  __syncthreads();
  // binned: the padding rows of every bin
  if (binned)
    for (long long i = tid; i < E * bin; i += kThreads) {
      const int e = static_cast<int>(i / bin), r = static_cast<int>(i - e * bin);
      if (r >= kept_s[e]) row_slot[i] = -1;
    }

  // ---- pass 2: counting-sort scatter, drop mask and the row maps; the loads
  // of 4 slots are issued before any of them is used.
  constexpr int kBatch = 4;
  for (int s0 = tid; s0 < S; s0 += kThreads * kBatch) {
    int ev[kBatch], rv[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int s = s0 + u * kThreads;
      ev[u] = s < S ? __ldg(idx + s) : -1;
      rv[u] = s < S ? __ldcg(rank_g + s) : 0;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int s = s0 + u * kThreads;
      if (s >= S) break;
      const int e = ev[u];
      if (e < 0 || e >= E) {
        slot_to_row[s] = -1;
        drop[s] = 1;
        continue;
      }
      const int r = rv[u];
      sorted_slot[start_s[e] + r] = s;
      const bool dr = r >= (binned ? bin : cap);
      drop[s] = dr ? 1 : 0;
      const int row = dr ? -1 : seg_s[e] + r;
      slot_to_row[s] = row;
      if (!dr) row_slot[row] = s;
    }
  }
  if (has_job) finish_aux_job(job, ctl, &hist[0][0]);  // the router's loss, left to this kernel
}

// ---------------------------------------------------------------- multi-CTA
// CTA b ranks the slots of its contiguous chunk [b*chunk, (b+1)*chunk) in slot
// order (the same warp-match / warp-scan scheme, over 8 warps), keeping each
// slot's expert and local rank in shared memory and publishing its per-expert
// counts. After one grid barrier every CTA adds, per expert, the counts of the
// CTAs before it (its rank offset) and of all CTAs (the histogram), takes the
// same block scan for bins / kept / seg_offsets, and scatters its own slots.
// Launched cooperatively, so all CTAs are resident; the barrier's spin is
// bounded and a time-out skips the scatter and sets MOE_DEVERR_TIMEOUT.
constexpr int kGThreads = 256;
constexpr int kGMaxChunk = 4096;


__global__ void __launch_bounds__(kGThreads)
permute_grid_kernel(const int32_t* __restrict__ idx, int S, int E, unsigned key_mask,
                    long long cap, int binned, int chunk, int32_t* __restrict__ counts,
                    int32_t* __restrict__ bins, int32_t* __restrict__ sorted_slot,
                    int32_t* __restrict__ slot_to_row, int32_t* __restrict__ row_slot,
                    uint8_t* __restrict__ drop, int32_t* __restrict__ kept,
                    int32_t* __restrict__ seg, int32_t* __restrict__ cta_counts, Control* ctl,
                    AuxJob job, int has_job) {
  pdl_begin();
  __shared__ __align__(16) int s_e[kGMaxChunk];
  __shared__ int s_rank[kGMaxChunk];
  __shared__ int hist[8][kMaxE + 1];
  __shared__ int running[kMaxE];
  __shared__ int pre[kMaxE];
  __shared__ int tot[kMaxE];
  __shared__ int start_s[kMaxE];
  __shared__ int seg_s[kMaxE + 1];
  __shared__ int kept_s[kMaxE];
  __shared__ int wtot_c[8], wtot_k[8];
  __shared__ int maxc_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt_mask = (1u << lane) - 1u;
  const int lo = blockIdx.x * chunk;
  const int hi = min(S, lo + chunk);

  for (int i = tid; i < 8 * (kMaxE + 1); i += kGThreads) (&hist[0][0])[i] = 0;
  for (int i = tid; i < kMaxE; i += kGThreads) { running[i] = 0; pre[i] = 0; tot[i] = 0; }
  if (tid == 0) maxc_s = 0;
  __syncthreads();

  // ---- local stable ranks of this CTA's slots
  for (int base = lo; base < hi; base += kGThreads) {
    const int s = base + tid;
    int e = -1;
    if (s < hi) {
      e = __ldg(idx + s);
      if (e < 0 || e >= E) {
        set_error(ctl, MOE_DEVERR_EXPERT_RANGE);
        e = -1;
      }
    }
    const unsigned key = e >= 0 ? (static_cast<unsigned>(e) & key_mask) : 0xffffffffu;
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    const int r_in_warp = __popc(peers & lt_mask);
    if (e >= 0 && lane == __ffs(peers) - 1) hist[warp][key] = __popc(peers);
    __syncthreads();
    for (int ke = tid; ke < E; ke += kGThreads) {
      int run = running[ke];
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const int c = hist[w][ke];
        hist[w][ke] = run;
        run += c;
      }
      running[ke] = run;
    }
    __syncthreads();
    if (s < hi) {
      s_e[s - lo] = e;
      s_rank[s - lo] = e >= 0 ? hist[warp][key] + r_in_warp : 0;
    }
    __syncthreads();
    for (int i = tid; i < 8 * E; i += kGThreads) hist[i / E][i % E] = 0;
    __syncthreads();
  }
  for (int e = tid; e < E; e += kGThreads)
    cta_counts[static_cast<size_t>(blockIdx.x) * E + e] = running[e];

  const bool ok = grid_barrier(ctl, gridDim.x);

  // ---- offsets of this CTA's ranks, and the histogram, from all CTAs' counts
  for (int i = tid; i < static_cast<int>(gridDim.x) * E; i += kGThreads) {
    const int b = i / E, e = i - b * E;
    const int c = __ldcg(cta_counts + i);
    atomicAdd(&tot[e], c);
    if (b < static_cast<int>(blockIdx.x)) atomicAdd(&pre[e], c);
  }
  __syncthreads();
  // counts, bins (inclusive), kept = min(count, C), seg (exclusive) over E <= 256;
  // binned layout: bin size C = cap, or the largest count when cap is none
  if (binned && cap == LLONG_MAX && tid < E) atomicMax(&maxc_s, tot[tid]);
  __syncthreads();
  const long long bin = binned ? (cap == LLONG_MAX ? static_cast<long long>(maxc_s) : cap) : 0;
  const long long lim = binned ? bin : cap;
  int c = 0, kp = 0, ci = 0, ki = 0;
  c = tid < E ? tot[tid] : 0;
  kp = static_cast<int>(c < lim ? c : lim);
  ci = c;
  ki = kp;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int n1 = __shfl_up_sync(0xffffffffu, ci, off);
    const int n2 = __shfl_up_sync(0xffffffffu, ki, off);
    if (lane >= off) { ci += n1; ki += n2; }
  }
  if (lane == 31) { wtot_c[warp] = ci; wtot_k[warp] = ki; }
  __syncthreads();
  int pc = 0, pk = 0;
  for (int w = 0; w < warp; ++w) { pc += wtot_c[w]; pk += wtot_k[w]; }
  ci += pc;
  ki += pk;
  if (tid < E) {
    const int sg = binned ? static_cast<int>(tid * bin) : ki - kp;
    if (blockIdx.x == 0) {
      counts[tid] = c;
      bins[tid] = ci;
      kept[tid] = kp;
      seg[tid] = sg;
    }
    start_s[tid] = ci - c;
    seg_s[tid] = sg;
    kept_s[tid] = kp;
  }
  if (tid == E - 1) {
    const int end = binned ? static_cast<int>(E * bin) : ki;
    if (blockIdx.x == 0) seg[E] = end;
    seg_s[E] = end;
  }
  __syncthreads();
  if (!ok) return;  // a timed-out barrier leaves the offsets unknown: write nothing
  // binned: this CTA's share of the padding rows of every bin
  if (binned)
    for (long long i = static_cast<long long>(blockIdx.x) * kGThreads + tid; i < E * bin;
         i += static_cast<long long>(gridDim.x) * kGThreads) {
      const int e = static_cast<int>(i / bin), r = static_cast<int>(i - e * bin);
      if (r >= kept_s[e]) row_slot[i] = -1;
    }

  // ---- counting-sort scatter, drop mask and the row maps
  for (int s = lo + tid; s < hi; s += kGThreads) {
    const int e = s_e[s - lo];
    if (e < 0) {
      slot_to_row[s] = -1;
      drop[s] = 1;
      continue;
    }
    const int r = s_rank[s - lo] + pre[e];
    const int pos = start_s[e] + r;
    if (pos < 0 || pos >= S) {  // only possible if the counts were corrupted
      set_error(ctl, MOE_DEVERR_ROW_RANGE);
      continue;
    }
    sorted_slot[pos] = s;
    const bool dr = r >= lim;
    drop[s] = dr ? 1 : 0;
    const int row = dr ? -1 : seg_s[e] + r;
    slot_to_row[s] = row;
    if (!dr) row_slot[row] = s;
  }
  if (has_job) finish_aux_job(job, ctl, s_e);  // the router's loss, spread over the CTAs
}

__global__ void set_wait_limit_kernel(Control* ctl, uint32_t limit_us) {
  pdl_begin();
  ctl->wait_limit_us = limit_us;
}

}  // namespace

cudaError_t launch_set_wait_limit(Control* ctl, uint32_t limit_us, cudaStream_t s) {
  return launch_pdl(set_wait_limit_kernel, dim3(1), dim3(1), 0, s, false, ctl, limit_us);
}

size_t permute_scratch_bytes(int T, int k, int E) {
  // rank scratch of the single-CTA kernel, then per-CTA counts of the multi-CTA one
  return align_up(static_cast<size_t>(T) * k * 4) + align_up(static_cast<size_t>(num_sms()) * E * 4);
}

static int key_mask_of(int E) {
  int bits = 1;
  while ((1 << bits) < E) ++bits;  // max(ceil(log2 E), 1)
  return static_cast<int>((1u << bits) - 1u);
}

cudaError_t launch_permute_single(const int32_t* idx, int T, int k, int E, int64_t cap,
                                  int32_t* counts, int32_t* bins, int32_t* sorted_slot,
                                  int32_t* slot_to_row, int32_t* row_slot, uint8_t* drop,
                                  int32_t* kept, int32_t* seg, int32_t* rank_scratch, Control* ctl,
                                  cudaStream_t s, bool binned, const AuxJob* aux_job) {
  const unsigned mask = static_cast<unsigned>(key_mask_of(E));
  const long long c = cap < 0 ? LLONG_MAX : static_cast<long long>(cap);
  const AuxJob job = aux_job != nullptr ? *aux_job : AuxJob{};
  return launch_pdl(permute_kernel, dim3(1), dim3(kThreads), 0, s, false, idx, T * k, E, mask, c,
                    binned ? 1 : 0, counts, bins, sorted_slot, slot_to_row, row_slot, drop, kept, seg, rank_scratch,
                    ctl, job, aux_job != nullptr ? 1 : 0);
}

bool permute_uses_grid(int T, int k, int E) {
  (void)E;
  const int S = T * k;
  const int g = std::max(1, std::min(num_sms(), (S + kGThreads - 1) / kGThreads));
  const int chunk = S > 0 ? (S + g - 1) / g : 0;
  return !(S == 0 || chunk > kGMaxChunk || g < 2);
}

cudaError_t launch_permute(const int32_t* idx, int T, int k, int E, int64_t cap, int32_t* counts,
                           int32_t* bins, int32_t* sorted_slot, int32_t* slot_to_row,
                           int32_t* row_slot, uint8_t* drop, int32_t* kept, int32_t* seg,
                           int32_t* scratch, Control* ctl, cudaStream_t s, bool binned,
                           const AuxJob* aux_job) {
  const int S = T * k;
  const int sms = num_sms();
  // enough CTAs that each chunk fits shared memory, at most one per SM, and
  // at least ~256 slots per CTA (the same rule as permute_uses_grid)
  const int g = std::max(1, std::min(sms, (S + kGThreads - 1) / kGThreads));
  const int chunk = S > 0 ? (S + g - 1) / g : 0;
  if (!permute_uses_grid(T, k, E))
    return launch_permute_single(idx, T, k, E, cap, counts, bins, sorted_slot, slot_to_row,
                                 row_slot, drop, kept, seg, scratch, ctl, s, binned, aux_job);
  int32_t* cta_counts = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(scratch) +
                                                   align_up(static_cast<size_t>(S) * 4));
  unsigned mask = static_cast<unsigned>(key_mask_of(E));
  long long c = cap < 0 ? LLONG_MAX : static_cast<long long>(cap);
  const AuxJob job = aux_job != nullptr ? *aux_job : AuxJob{};
  return launch_pdl(permute_grid_kernel, dim3(g), dim3(kGThreads), 0, s, true, idx, S, E, mask, c,
                    binned ? 1 : 0, chunk, counts, bins, sorted_slot, slot_to_row, row_slot, drop, kept, seg,
                    cta_counts, ctl, job, aux_job != nullptr ? 1 : 0);
}

}  // namespace moe
