// Internal declarations shared by the kernels and the C-ABI layer.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <cstddef>
#include <cuda.h>

#include "../../include/moe_b200.h"

namespace moe {

// First 256 bytes of every workspace.
struct Control {
  uint32_t err;           // MOE_DEVERR_* bits, sticky until cleared
  uint32_t route_ticket;  // blocks of the router that finished (reset by the last one)
  uint32_t bar_count;     // grid barrier: blocks arrived (reset by the last one)
  uint32_t bar_gen;       // grid barrier: generation, bumped when all arrived
  uint32_t wait_limit_us; // limit of the waits between CTAs; 0: 2 s
  uint32_t gemm_next;     // CTA-pair GEMM: next work unit (reset by the last pair)
  uint32_t gemm_done;     // CTA-pair GEMM: pairs that finished (reset by the last pair)
  uint32_t reserved[57];
};
static_assert(sizeof(Control) == 256, "control block is 256 bytes");

constexpr size_t kAlign = 256;
__host__ __device__ inline size_t align_up(size_t v, size_t a = kAlign) { return (v + a - 1) / a * a; }

__device__ __forceinline__ void set_error(Control* ctl, uint32_t bits) {
  atomicOr(&ctl->err, bits);
}

// How long a wait between CTAs may last before it gives up (ns).
__device__ __forceinline__ uint64_t wait_limit_ns(const Control* ctl) {
  const uint32_t us = *reinterpret_cast<const volatile uint32_t*>(&ctl->wait_limit_us);
  return us == 0 ? 2000000000ull : static_cast<uint64_t>(us) * 1000ull;
}

__device__ __forceinline__ float bf16_to_f32(uint16_t u) {
  return __uint_as_float(static_cast<uint32_t>(u) << 16);
}

template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f32(float v) { return v; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
};

// The load-balance loss's last step, which a layer forward may leave to the
// permute kernel (it runs next anyway) when the router would otherwise need a
// launch of its own for it: aux = E * sum_e (c_e / (T k)) (p_e / T)
// from the router's per-block partials part_p / part_c [E][ldb] (nblk
// blocks), and the z-loss, mean over tokens of lse^2, from part_z [nblk]
// (null: none). terms [E] is scratch.
struct AuxJob {
  int pending;  // 1: launch_route left the step to a later kernel
  const float* part_p;
  const int32_t* part_c;
  const float* part_z;
  double* terms;
  float* aux;
  float* z;
  int ldb, nblk, E, T, k;
};

// Finish a deferred load-balance loss with the first min(gridDim.x, E) CTAs
// of a grid (every thread of each CTA calls it; threads 0..255 do the work,
// blockDim.x >= 256; the other CTAs return at once). CTA b takes the experts
// b, b + gridDim.x, ...: thread i adds the partials of blocks i, i + 256, ...
// in float64, each warp reduces with a fixed butterfly and thread 0 adds the
// 8 warp sums in order; the last of those CTAs (ticket) adds the E terms the
// same way and reduces the z-loss likewise. Deterministic. Uses
// ctl->route_ticket (free during the permute).
constexpr int kAuxFinishThreads = 256;

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

__device__ __forceinline__ long long warp_sum_i64(long long v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// scratch: >= 2 * 8 * 8 bytes of the caller's shared memory, 8-byte aligned,
// free from this call on (a barrier first orders it after the caller's use).
__device__ __forceinline__ void finish_aux_job(const AuxJob& j, Control* ctl, void* scratch) {
  constexpr int nt = kAuxFinishThreads, nw = nt / 32;
  const int parts = min(static_cast<int>(gridDim.x), j.E);
  if (static_cast<int>(blockIdx.x) >= parts) return;  // CTA-uniform
  double* wp = static_cast<double*>(scratch);         // [nw]
  long long* wc = reinterpret_cast<long long*>(wp + nw);  // [nw]
  double* wz = wp + nw;                                   // [nw], the z-loss step (reuses wc)
  __shared__ int fa_last;
  const int tid = threadIdx.x, lane = tid & 31, wq = tid >> 5;
  const bool part = tid < nt;
  __syncthreads();
  for (int e = blockIdx.x; e < j.E; e += gridDim.x) {
    if (part) {
      double ps = 0.0;
      long long cs = 0;
      for (int b = tid; b < j.nblk; b += nt) {
        ps += static_cast<double>(__ldcg(j.part_p + static_cast<size_t>(e) * j.ldb + b));
        cs += __ldcg(j.part_c + static_cast<size_t>(e) * j.ldb + b);
      }
      ps = warp_sum_f64(ps);
      cs = warp_sum_i64(cs);
      if (lane == 0) { wp[wq] = ps; wc[wq] = cs; }
    }
    __syncthreads();
    if (tid == 0) {
      double p = 0.0;
      long long c = 0;
      for (int w = 0; w < nw; ++w) { p += wp[w]; c += wc[w]; }
      j.terms[e] = j.T > 0 ? (static_cast<double>(c) / (static_cast<double>(j.T) * j.k)) * (p / j.T) : 0.0;
    }
    __syncthreads();
  }
  if (tid == 0) {
    __threadfence();
    fa_last = atomicAdd(&ctl->route_ticket, 1u) == static_cast<unsigned>(parts) - 1u;
  }
  __syncthreads();
  if (!fa_last) return;
  __threadfence();
  if (part) {
    double v = tid < j.E ? __ldcg(j.terms + tid) : 0.0;
    v = warp_sum_f64(v);
    double zs = 0.0;
    if (j.part_z != nullptr)
      for (int b = tid; b < j.nblk; b += nt) zs += static_cast<double>(__ldcg(j.part_z + b));
    zs = warp_sum_f64(zs);
    if (lane == 0) { wp[wq] = v; wz[wq] = zs; }
  }
  __syncthreads();
  if (tid == 0) {
    double tot = 0.0, z = 0.0;
    for (int w = 0; w < nw; ++w) { tot += wp[w]; z += wz[w]; }
    *j.aux = static_cast<float>(j.E * tot);
    if (j.part_z != nullptr) *j.z = j.T > 0 ? static_cast<float>(z / j.T) : 0.f;
    ctl->route_ticket = 0u;
  }
}

// ------------------------------------------- programmatic dependent launch
// Every kernel of the library is launched with programmatic stream
// serialisation and starts with pdl_begin(): it waits there until the
// previous kernel on the stream has finished and its writes are visible
// (griddepcontrol.wait; a no-op when launched without the attribute), then
// lets the next kernel be scheduled. The next kernel's launch and block
// scheduling thus overlap this kernel's run instead of following its end.
// A dependent grid is launched only after every block of this grid has
// started, so its waiting blocks never hold resources this grid still needs.
__device__ __forceinline__ void pdl_begin() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns_c() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Barrier over all blocks of a cooperatively launched grid (every block is
// resident), through bar_count / bar_gen of the control block: the last block
// to arrive resets the count and bumps the generation. The spin is bounded by
// the control block's wait limit; a time-out sets MOE_DEVERR_TIMEOUT and
// returns false in every thread of the block.
__device__ __forceinline__ bool grid_barrier(Control* ctl, unsigned nblocks) {
  __shared__ int ok_s;
  __threadfence();  // this thread's global writes are visible before the block arrives
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    __threadfence();
    volatile unsigned* gen_p = &ctl->bar_gen;
    const unsigned gen = *gen_p;
    const unsigned arrived = atomicAdd(&ctl->bar_count, 1u);
    if (arrived == nblocks - 1) {
      ctl->bar_count = 0u;
      __threadfence();
      atomicAdd(&ctl->bar_gen, 1u);
    } else {
      const uint64_t limit = wait_limit_ns(ctl);
      const uint64_t t0 = globaltimer_ns_c();
      while (*gen_p == gen) {
        if (globaltimer_ns_c() - t0 > limit) {
          set_error(ctl, MOE_DEVERR_TIMEOUT);
          ok = 0;
          break;
        }
        __nanosleep(64);
      }
    }
    __threadfence();
    ok_s = ok;
  }
  __syncthreads();
  return ok_s != 0;
}

// Counts every kernel this library launches (moe_kernel_launches reads it).
void note_launch();

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       bool cooperative, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cooperative ? 2 : 1;
  note_launch();
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// launch_pdl for a kernel launched in clusters of cluster_x CTAs along x
// (grid.x a multiple of cluster_x; 1 = no cluster).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                               cudaStream_t s, int cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(cluster_x);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster_x > 1 ? 2 : 1;
  note_launch();
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ------------------------------------------------------------------ launchers
// Router.
size_t route_partials_bytes(int T, int E);
// noise: optional [T, E] fp32 added to the logits after the bias; z_out:
// optional z-loss output (mean over tokens of the squared log-sum-exp);
// temperature: the softmax sees logits / temperature (> 0; 1 = plain).
cudaError_t launch_route(const void* x, const void* wg, const float* bias, const float* noise,
                         moe_dtype_t dt, int T, int d, int E, int k, int32_t* idx, float* w,
                         float* aux, float* z_out, float* logits, float* probs,
                         float* logits_scratch, void* partials, Control* ctl, cudaStream_t s,
                         float temperature = 1.0f, AuxJob* defer_aux = nullptr);
size_t route_logits_scratch_bytes(int T, int d, int E);
// Router backward (see router_backward.cu): d_logits [T, E] fp32 (or NULL:
// kept in scratch), dx [T, d] (dtype) or NULL, d_wg [d, E] fp32 or NULL.
// logits (before the temperature) are read only when d_z != 0; counts of the
// picks are taken on the device when d_aux != 0.
size_t route_backward_scratch_bytes(int T, int d, int E);
cudaError_t launch_route_backward(const void* x, const void* wg, moe_dtype_t dt, int T, int d,
                                  int E, int k, const float* probs, const float* logits,
                                  const int32_t* idx, const float* w, const float* d_w,
                                  float d_aux, float d_z, float temperature, float* d_logits,
                                  void* dx, float* d_wg, void* scratch, Control* ctl,
                                  cudaStream_t s);

// Permute. launch_permute picks the multi-CTA kernel when the slots fit its
// per-CTA shared memory, else the single-CTA kernel; launch_permute_single
// always runs the single-CTA kernel (needs only the rank scratch). binned:
// the [E, C] bucket layout (row e*C + rank; C = cap, or the largest count
// when cap < 0; padding rows get row_slot -1).
size_t permute_scratch_bytes(int T, int k, int E);
// Whether launch_permute runs the multi-CTA kernel for these sizes (which
// finishes a deferred load-balance loss cheaply across its CTAs).
bool permute_uses_grid(int T, int k, int E);
cudaError_t launch_permute_single(const int32_t* idx, int T, int k, int E, int64_t cap,
                                  int32_t* counts, int32_t* bins, int32_t* sorted_slot,
                                  int32_t* slot_to_row, int32_t* row_slot, uint8_t* drop,
                                  int32_t* kept, int32_t* seg, int32_t* rank_scratch, Control* ctl,
                                  cudaStream_t s, bool binned = false,
                                  const AuxJob* aux_job = nullptr);
// aux_job: a load-balance loss left by launch_route to finish (see AuxJob).
cudaError_t launch_permute(const int32_t* idx, int T, int k, int E, int64_t cap, int32_t* counts,
                           int32_t* bins, int32_t* sorted_slot, int32_t* slot_to_row,
                           int32_t* row_slot, uint8_t* drop, int32_t* kept, int32_t* seg,
                           int32_t* rank_scratch, Control* ctl, cudaStream_t s,
                           bool binned = false, const AuxJob* aux_job = nullptr);

// Router training inputs (noise.cu): x' = x * uniform(1 - eps, 1 + eps)
// elementwise (n elements, dtype dt), and std * N(0, 1) logit noise (n
// values, fp32), both from Philox4x32-10 keyed by seed.
cudaError_t launch_jitter(const void* x, moe_dtype_t dt, long long n, float eps, uint64_t seed,
                          void* out, cudaStream_t s);
cudaError_t launch_logit_noise(long long n, float std, uint64_t seed, float* out, cudaStream_t s);

// Gather. binned: rows with row_slot -1 are padding and are written as zeros.
// zero_out (with slot_to_row [T, k]): also zero the [T, d] output rows of
// tokens none of whose slots was kept (the combine runs in the down
// projection). x_perm NULL: only that zeroing.
cudaError_t launch_gather(const void* x, size_t elem, int T, int d, int k, const int32_t* row_slot,
                          const int32_t* seg, int E, int64_t rows_max, void* x_perm, Control* ctl,
                          cudaStream_t s, bool binned = false, const int32_t* slot_to_row = nullptr,
                          void* zero_out = nullptr);

// Control block: write the wait limit (one thread).
cudaError_t launch_set_wait_limit(Control* ctl, uint32_t limit_us, cudaStream_t s);

// Grouped GEMMs. bf16: A is x_perm [rows_max, d] when row_slot is NULL, else
// the token rows x [a_rows = T, d], gathered by the up projection itself
// (row r reads token row_slot[r] / k). Expert e's rows start at seg[e]; there
// are kept[e] of them (binned layout), or seg[e + 1] - seg[e] when kept is NULL.
// The combine folded into the down projection (k = 1): each row's output,
// scaled by w[slot], goes to out[slot / k]; y is not written.
struct CombineOut {
  const int32_t* row_slot;  // [rows_max] slot of each row (-1: binned padding)
  const float* w;           // [T * k] top-k weights
  void* out;                // [T, d] layer output
  int T;
};
// slots: rows the permute distributes over the experts (T * k), which picks
// the single-CTA or the CTA-pair kernel; negative: rows_max.
cudaError_t launch_ffn_bf16(const void* a, int64_t a_rows, const int32_t* row_slot, int k,
                            const void* w1, const void* w3, const void* w2, moe_act_t act,
                            int64_t rows_max, int d, int F, int E, const int32_t* seg,
                            const int32_t* kept, void* h, void* y, Control* ctl, cudaStream_t s,
                            cudaEvent_t after_up, const CombineOut* comb = nullptr,
                            int64_t slots = -1);
cudaError_t launch_ffn_f32(const float* x_perm, const float* w1, const float* w3, const float* w2,
                           moe_act_t act, int64_t rows_max, int d, int F, int E,
                           const int32_t* seg, float* h, float* y, Control* ctl, cudaStream_t s,
                           cudaEvent_t after_up);

// Combine.
cudaError_t launch_combine(const void* y, const float* w, const int32_t* slot_to_row, size_t elem,
                           int T, int d, int k, int64_t rows_max, void* out, Control* ctl,
                           cudaStream_t s);

// Expert-parallel dispatch plans (ep.cu). Experts are owned in contiguous
// blocks of e_loc per rank.
cudaError_t launch_ep_send_plan(const int32_t* kept, const int32_t* seg, int world, int e_loc,
                                int32_t* send_rows, int32_t* send_offsets, Control* ctl,
                                cudaStream_t s);
cudaError_t launch_ep_recv_plan(const int32_t* counts, int world, int e_loc, long long rows_cap,
                                int32_t* recv_rows, int32_t* recv_offsets, int32_t* local_seg,
                                int32_t* local_to_recv, int32_t* recv_to_local, Control* ctl,
                                cudaStream_t s);

int num_sms();

// 2-D bf16 TMA map over [rows, cols] row-major, box [box_rows, 64 cols], 128-byte swizzle.
bool make_tma_2d_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                      uint32_t box_rows);
// Box [box_rows, box_cols] without swizzle (rows land back to back).
bool make_tma_2d_bf16_plain(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                            uint32_t box_cols, uint32_t box_rows);
// The same with a row stride of ld elements (ld * 2 a multiple of 16 bytes).
bool make_tma_2d_bf16_ld(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                         uint32_t box_rows);

}  // namespace moe
