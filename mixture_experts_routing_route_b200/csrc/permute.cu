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
#include <climits>

namespace moe {

namespace {

constexpr int kThreads = 1024;
constexpr int kMaxE = 256;

__global__ void __launch_bounds__(kThreads)
permute_kernel(const int32_t* __restrict__ idx, int S, int E, unsigned key_mask, long long cap,
               int32_t* __restrict__ counts, int32_t* __restrict__ bins,
               int32_t* __restrict__ sorted_slot, int32_t* __restrict__ slot_to_row,
               int32_t* __restrict__ row_slot, uint8_t* __restrict__ drop,
               int32_t* __restrict__ kept, int32_t* __restrict__ seg, int32_t* __restrict__ rank_g,
               Control* ctl) {
  __shared__ int hist[32][kMaxE + 1];
  __shared__ int running[kMaxE];
  __shared__ int start_s[kMaxE];
  __shared__ int seg_s[kMaxE + 1];
  __shared__ int wtot_c[8], wtot_k[8];
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const unsigned lt_mask = (1u << lane) - 1u;

  for (int i = tid; i < 32 * (kMaxE + 1); i += kThreads) (&hist[0][0])[i] = 0;
  for (int i = tid; i < kMaxE; i += kThreads) running[i] = 0;
  __syncthreads();

  // ---- pass 1: stable rank of every slot within its expert
  for (int base = 0; base < S; base += kThreads) {
    const int s = base + tid;
    int e = -1;
    if (s < S) {
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
  int c = 0, kp = 0, ci = 0, ki = 0;
  if (tid < 256) {
    c = tid < E ? running[tid] : 0;
    kp = static_cast<int>(c < cap ? c : cap);
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
      counts[tid] = c;
      bins[tid] = ci;
      kept[tid] = kp;
      seg[tid] = ki - kp;
      start_s[tid] = ci - c;
      seg_s[tid] = ki - kp;
    }
    if (tid == E - 1) { seg[E] = ki; seg_s[E] = ki; }
  }
  __syncthreads();

  // ---- pass 2: counting-sort scatter, drop mask and the row maps
  for (int s = tid; s < S; s += kThreads) {
    const int e = __ldg(idx + s);
    if (e < 0 || e >= E) {
      slot_to_row[s] = -1;
      drop[s] = 1;
      continue;
    }
    const int r = rank_g[s];
    sorted_slot[start_s[e] + r] = s;
    const bool dr = r >= cap;
    drop[s] = dr ? 1 : 0;
    const int row = dr ? -1 : seg_s[e] + r;
    slot_to_row[s] = row;
    if (!dr) row_slot[row] = s;
  }
}

}  // namespace

size_t permute_scratch_bytes(int T, int k, int E) {
  (void)E;
  return align_up(static_cast<size_t>(T) * k * 4);
}

cudaError_t launch_permute(const int32_t* idx, int T, int k, int E, int64_t cap, int32_t* counts,
                           int32_t* bins, int32_t* sorted_slot, int32_t* slot_to_row,
                           int32_t* row_slot, uint8_t* drop, int32_t* kept, int32_t* seg,
                           int32_t* rank_scratch, Control* ctl, cudaStream_t s) {
  int bits = 1;
  while ((1 << bits) < E) ++bits;  // max(ceil(log2 E), 1)
  const unsigned mask = (1u << bits) - 1u;
  const long long c = cap < 0 ? LLONG_MAX : static_cast<long long>(cap);
  permute_kernel<<<1, kThreads, 0, s>>>(idx, T * k, E, mask, c, counts, bins, sorted_slot,
                                        slot_to_row, row_slot, drop, kept, seg, rank_scratch, ctl);
  return cudaGetLastError();
}

}  // namespace moe
