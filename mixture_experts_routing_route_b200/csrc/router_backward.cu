// Router backward: gradients of the router's losses through the tempered
// softmax and the gate ("ops-transformer MoE operators", 实现: the gating
// operator carries the router's forward and its backward; 坑3: gradients
// reach the experts through the softmax). For the scalar
//
//   L = sum_{t,j} d_w[t, j] * w[t, j] + d_aux * aux + d_z * z
//
// (w: renormalised top-k weights, aux = E sum_i f_i P_i, z = mean_t lse_t^2
// of l / tau), with the pick and the counts f_i held fixed:
//
//   dL/dp_{i_j}  = (d_w[t, j] - sum_m d_w[t, m] w[t, m]) / s_t,  s_t = sum_j p_{i_j}
//   dL/dp[t, e] += d_aux * E * f_e / T
//   dL/dl[t, e]  = p_e (dL/dp_e - sum_i p_i dL/dp_i) / tau
//                  + d_z * (2 / T) * lse_t * p_e / tau
//   dx  = dL/dl Wg^T        dWg = x^T dL/dl
//
// Kernels: d_logits (fp32) by a warp per token after an expert histogram of
// the picks (f, when d_aux != 0) for small T, or by a thread per token that
// counts the picks in the same launch for large T. The two T x d passes run
// on the tensor cores for bf16 with E <= 64 (bwd_dx_tc, bwd_dwg_tc: d_logits
// enters as bf16 hi + lo terms, products summed in fp32), otherwise on CUDA
// cores in fp32 (bwd_dx; bwd_dwg_part + bwd_dwg_reduce). dWg is a sum of
// partials added in a fixed order (deterministic); dx is rounded once to the
// input dtype.
#include "common.cuh"
#include "ptx.cuh"

#include <cmath>

namespace moe {
namespace {

constexpr unsigned kFull = 0xffffffffu;

// counts[e] = slots that picked expert e (before any drop). One block up to
// kHistOneBlock picks (the ticket's round trip costs more than a second block
// saves there: Mixtral router backward 27.8 against 29.7 us); above, block b counts
// its share of the picks (per_block4 16-byte loads of 4 picks each; the last
// block also the S % 4 tail) in shared memory and writes them as partial b;
// the last block to finish (the control block's route_ticket, which it
// resets) adds the partials in block order. Deterministic (integers).
constexpr int kHistThreads = 1024;
constexpr int kHistMaxBlocks = 64;
constexpr long long kHistOneBlock = 16384;

__global__ void __launch_bounds__(kHistThreads)
bwd_hist(const int32_t* __restrict__ idx, long long S, int E, long long per_block4,
         int32_t* __restrict__ part, int32_t* __restrict__ counts, Control* ctl) {
  pdl_begin();
  __shared__ int h[256];  // E <= 256
  __shared__ int last_s;
  for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
  __syncthreads();
  auto add = [&](int e) {
    if (e < 0 || e >= E) set_error(ctl, MOE_DEVERR_EXPERT_RANGE);
    else atomicAdd(&h[e], 1);
  };
  // four picks per 16-byte load (idx is 16-byte aligned), then the tail
  const long long S4 = S / 4;
  const long long q0 = static_cast<long long>(blockIdx.x) * per_block4;
  const long long q1 = min(S4, q0 + per_block4);
  for (long long q = q0 + threadIdx.x; q < q1; q += blockDim.x) {
    const int4 v = __ldg(reinterpret_cast<const int4*>(idx) + q);
    add(v.x);
    add(v.y);
    add(v.z);
    add(v.w);
  }
  if (blockIdx.x == gridDim.x - 1)
    for (long long s = S4 * 4 + threadIdx.x; s < S; s += blockDim.x) add(__ldg(idx + s));
  __syncthreads();
  if (gridDim.x == 1) {  // one block: the counts directly
    for (int e = threadIdx.x; e < E; e += blockDim.x) counts[e] = h[e];
    return;
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) part[static_cast<size_t>(blockIdx.x) * E + e] = h[e];
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last_s = atomicAdd(&ctl->route_ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!last_s) return;
  __threadfence();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int n = 0;
    for (unsigned b = 0; b < gridDim.x; ++b) n += __ldcg(part + static_cast<size_t>(b) * E + e);
    counts[e] = n;
  }
  if (threadIdx.x == 0) ctl->route_ticket = 0u;
}

constexpr int kLogitWarps = 16;

// Warp per token; lane holds experts lane + 32 q, q < EPL. The short per-lane
// chains and a grid over every SM suit small T (counts from bwd_hist first);
// with dlT set (E <= 64) it also writes the bf16 terms of d_logits for the
// tensor-core dWg, and block 0 zeroes dWg's tickets. A block's 16 warps take
// 16 consecutive tokens per round, so with dlT the round's terms are staged
// in shared memory and each dlT row gets one whole 32-byte sector per round
// (ldt is a multiple of 16) instead of a 2-byte store per lane and row.
template <int EPL>
__global__ void __launch_bounds__(kLogitWarps * 32)
bwd_logits(const float* __restrict__ probs, const float* __restrict__ logits,
           const int32_t* __restrict__ idx, const float* __restrict__ w,
           const float* __restrict__ d_w, const int32_t* __restrict__ counts, float d_aux,
           float d_z, float inv_tau, int T, int E, int k, float* __restrict__ d_logits,
           __nv_bfloat16* __restrict__ dlT, int ec, int ldt, int* __restrict__ tickets,
           int ntickets, Control* ctl) {
  pdl_begin();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (tickets != nullptr && blockIdx.x == 0)
    for (int i = threadIdx.x; i < ntickets; i += blockDim.x) tickets[i] = 0;
  // the aux term is the same for every token: d_aux * E * f_e / T
  float aux_c[EPL];
#pragma unroll
  for (int q = 0; q < EPL; ++q) {
    const int e = lane + 32 * q;
    aux_c[q] = 0.f;
    if (counts != nullptr && e < E)
      aux_c[q] = d_aux * static_cast<float>(E) *
                 (static_cast<float>(__ldg(counts + e)) / (static_cast<float>(T) * k)) /
                 static_cast<float>(T);
  }
  const float zc = d_z * 2.0f / static_cast<float>(T);
  __shared__ __align__(16) __nv_bfloat16 st_s[128][kLogitWarps];  // [hi/lo row][token of the round]
  // block-uniform rounds (the dlT staging has barriers)
  for (long long base = static_cast<long long>(blockIdx.x) * kLogitWarps; base < T;
       base += static_cast<long long>(gridDim.x) * kLogitWarps) {
    const int t = static_cast<int>(base) + warp;
    if (t >= T) {
      if (dlT != nullptr)
        for (int n = lane; n < 2 * ec; n += 32) st_s[n][warp] = __float2bfloat16_rn(0.f);
    } else {
    const size_t row = static_cast<size_t>(t) * E;
    float p[EPL], dp[EPL];
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
      const int e = lane + 32 * q;
      p[q] = e < E ? __ldg(probs + row + e) : 0.f;
      dp[q] = aux_c[q];
    }
    if (d_w != nullptr) {
      // lane j < k: pick j's expert, weight, upstream gradient and probability
      int ej = 0;
      float gj = 0.f, wj = 0.f, pj = 0.f;
      if (lane < k) {
        ej = __ldg(idx + static_cast<size_t>(t) * k + lane);
        if (ej < 0 || ej >= E) {
          set_error(ctl, MOE_DEVERR_EXPERT_RANGE);
          ej = 0;
        }
        gj = __ldg(d_w + static_cast<size_t>(t) * k + lane);
        wj = __ldg(w + static_cast<size_t>(t) * k + lane);
        pj = __ldg(probs + row + ej);
      }
      float s = pj, gw = gj * wj;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) {
        s += __shfl_xor_sync(kFull, s, off);
        gw += __shfl_xor_sync(kFull, gw, off);
      }
      const float val = (gj - gw) / s;
      for (int j = 0; j < k; ++j) {  // the owner of pick j's expert adds its term
        const int e = __shfl_sync(kFull, ej, j);
        const float v = __shfl_sync(kFull, val, j);
        if (lane == (e & 31)) {
#pragma unroll
          for (int q = 0; q < EPL; ++q)
            if (q == (e >> 5)) dp[q] += v;
        }
      }
    }
    float c = 0.f;
#pragma unroll
    for (int q = 0; q < EPL; ++q) c += p[q] * dp[q];
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) c += __shfl_xor_sync(kFull, c, off);
    float dl[EPL];
#pragma unroll
    for (int q = 0; q < EPL; ++q) dl[q] = p[q] * (dp[q] - c) * inv_tau;
    if (logits != nullptr) {  // z-loss term: lse of l / tau
      float lt[EPL], m = -INFINITY;
#pragma unroll
      for (int q = 0; q < EPL; ++q) {
        const int e = lane + 32 * q;
        lt[q] = e < E ? __ldg(logits + row + e) * inv_tau : -INFINITY;
        m = fmaxf(m, lt[q]);
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
      float se = 0.f;
#pragma unroll
      for (int q = 0; q < EPL; ++q) se += (lane + 32 * q < E) ? expf(lt[q] - m) : 0.f;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) se += __shfl_xor_sync(kFull, se, off);
      const float lse = m + logf(se);
#pragma unroll
      for (int q = 0; q < EPL; ++q) dl[q] += zc * lse * p[q] * inv_tau;
    }
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
      const int e = lane + 32 * q;
      if (e < E) d_logits[row + e] = dl[q];
    }
    if (dlT != nullptr) {
      // the tensor-core dWg's B operand (E <= 64): dlT[e][t] = hi,
      // dlT[ec + e][t] = lo for the lane's experts e = lane + 32 q < ec
#pragma unroll
      for (int q = 0; q < EPL; ++q) {
        const int e = lane + 32 * q;
        if (e < ec) {
          const float v = e < E ? dl[q] : 0.f;
          const __nv_bfloat16 h = __float2bfloat16_rn(v);
          st_s[e][warp] = h;
          st_s[ec + e][warp] = __float2bfloat16_rn(v - __bfloat162float(h));
        }
      }
    }
    }
    if (dlT != nullptr) {
      __syncthreads();
      // row n, tokens base .. base + 15: two 16-byte stores
      for (int i = threadIdx.x; i < 4 * ec; i += kLogitWarps * 32) {
        const int n = i >> 1, h = i & 1;
        *reinterpret_cast<uint4*>(dlT + static_cast<size_t>(n) * ldt + base + 8 * h) =
            *reinterpret_cast<const uint4*>(&st_s[n][8 * h]);
      }
      __syncthreads();
    }
  }
}

// EC fp32 values of row t of a [T][E] array (t < T), zeros past E; one or
// more 16-byte loads when E == EC (rows 16-byte aligned).
template <int EC>
__device__ __forceinline__ void load_row_f32(const float* __restrict__ a, long long t, int E, float (&v)[EC]) {
  if (E == EC) {
    const float4* p = reinterpret_cast<const float4*>(a + t * EC);
#pragma unroll
    for (int i = 0; i < EC / 4; ++i) {
      const float4 q = __ldg(p + i);
      v[4 * i] = q.x; v[4 * i + 1] = q.y; v[4 * i + 2] = q.z; v[4 * i + 3] = q.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < EC; ++e) v[e] = e < E ? __ldg(a + t * E + e) : 0.f;
  }
}

// d_logits with a thread per token, for large T (E <= 16, k <= 8; EC = 8
// or 16 register slots, zeros past E): the token's probabilities, logits,
// picks, weights and upstream gradients are loaded together as whole rows, so
// a thread waits on memory once and every load of a warp is one contiguous
// range. With the aux term (count) each block first counts its own tokens'
// picks (per-lane 8-bit counters packed four to a word, flushed before they
// can carry, then one warp reduction per expert) and publishes them; after
// one grid barrier (cooperative launch: every block is resident; the wait is
// bounded) every block adds all blocks' counts in block order, so no separate
// histogram launch is needed. With dlT set it also writes the bf16 terms of
// d_logits, transposed, for the tensor-core dWg: dlT[e][t] = hi,
// dlT[EC + e][t] = lo (consecutive tokens: coalesced), and block 0 zeroes
// dWg's tickets.
constexpr int kTptThreads = 256;
constexpr int kTptMaxBlocks = 1024;        // hist_part holds kTptMaxBlocks x 16 counts
constexpr int kTptMaxK = 8;
constexpr long long kTptMinPicks = 16384;  // below this many picks the warp kernels are faster

// one lane's picks into 8-bit counters, four experts per word
template <int EC>
__device__ __forceinline__ void tally(int e, int E, Control* ctl, uint32_t (&pk)[EC / 4]) {
  if (e < 0 || e >= E) {
    set_error(ctl, MOE_DEVERR_EXPERT_RANGE);
    return;
  }
  const uint32_t inc = 1u << ((e & 3) * 8);
#pragma unroll
  for (int q = 0; q < EC / 4; ++q) pk[q] += (e >> 2) == q ? inc : 0u;
}

template <int EC>
__global__ void __launch_bounds__(kTptThreads)
bwd_logits_tpt(const float* __restrict__ probs, const float* __restrict__ logits,
               const int32_t* __restrict__ idx, const float* __restrict__ w,
               const float* __restrict__ d_w, int count, int32_t* __restrict__ hist_part,
               float d_aux, float d_z, float inv_tau, int T, int E, int k,
               float* __restrict__ d_logits, __nv_bfloat16* __restrict__ dlT, int ldt,
               int* __restrict__ tickets, int ntickets, Control* ctl) {
  pdl_begin();
  __shared__ int h_s[EC];
  __shared__ float aux_s[EC];
  const int tid = threadIdx.x, lane = tid & 31;
  if (tickets != nullptr && blockIdx.x == 0)
    for (int i = tid; i < ntickets; i += kTptThreads) tickets[i] = 0;
  if (tid < EC) {
    h_s[tid] = 0;
    aux_s[tid] = 0.f;
  }
  const long long stride = static_cast<long long>(gridDim.x) * kTptThreads;
  long long t = static_cast<long long>(blockIdx.x) * kTptThreads + tid;
  // the current token's inputs, loaded before they are needed
  float ip[EC], ilt[EC], ig[kTptMaxK], iw[kTptMaxK];
  int ie[kTptMaxK];
  auto load = [&](long long u) {
    load_row_f32<EC>(probs, u, E, ip);
    if (logits != nullptr) load_row_f32<EC>(logits, u, E, ilt);
#pragma unroll
    for (int j = 0; j < kTptMaxK; ++j) {
      const bool on = d_w != nullptr && j < k;
      ie[j] = on ? __ldg(idx + u * k + j) : 0;
      ig[j] = on ? __ldg(d_w + u * k + j) : 0.f;
      iw[j] = on ? __ldg(w + u * k + j) : 0.f;
    }
  };
  if (t < T) load(t);
  __syncthreads();
  if (count) {
    uint32_t pk[EC / 4];
#pragma unroll
    for (int q = 0; q < EC / 4; ++q) pk[q] = 0u;
    // this block's tokens: at most 255 picks per lane between flushes
    int n_since = 0;
    for (long long u = t; u < T; u += stride) {
      for (int j = 0; j < k; ++j) tally<EC>(__ldg(idx + u * k + j), E, ctl, pk);
      n_since += k;
      if (n_since > 255 - kTptMaxK) {
#pragma unroll
        for (int e = 0; e < EC; ++e) {
          const uint32_t c = (pk[e >> 2] >> ((e & 3) * 8)) & 0xffu;
          if (c != 0) atomicAdd(&h_s[e], static_cast<int>(c));
        }
#pragma unroll
        for (int q = 0; q < EC / 4; ++q) pk[q] = 0u;
        n_since = 0;
      }
    }
#pragma unroll
    for (int e = 0; e < EC; ++e) {
      const unsigned c = __reduce_add_sync(kFull, (pk[e >> 2] >> ((e & 3) * 8)) & 0xffu);
      if (lane == 0 && c != 0) atomicAdd(&h_s[e], static_cast<int>(c));
    }
    __syncthreads();
    if (tid < EC) hist_part[static_cast<size_t>(blockIdx.x) * EC + tid] = h_s[tid];
    if (!grid_barrier(ctl, gridDim.x)) return;
    if (tid < EC) {
      int n = 0;
      for (unsigned b = 0; b < gridDim.x; ++b) n += __ldcg(hist_part + static_cast<size_t>(b) * EC + tid);
      h_s[tid] = n;
    }
    __syncthreads();
    // the aux term is the same for every token: d_aux * E * f_e / T
    if (tid < EC)
      aux_s[tid] = tid < E ? d_aux * static_cast<float>(E) *
                                 (static_cast<float>(h_s[tid]) / (static_cast<float>(T) * k)) /
                                 static_cast<float>(T)
                           : 0.f;
    __syncthreads();
  }
  const float zc = d_z * 2.0f / static_cast<float>(T);
  while (t < T) {
    float dp[EC];
#pragma unroll
    for (int e = 0; e < EC; ++e) dp[e] = aux_s[e];
    if (d_w != nullptr) {
      float s = 0.f, gw = 0.f;
#pragma unroll
      for (int j = 0; j < kTptMaxK; ++j) {
        if (j < k) {
          if (ie[j] < 0 || ie[j] >= E) {
            set_error(ctl, MOE_DEVERR_EXPERT_RANGE);
            ie[j] = 0;
          }
          float pj = 0.f;
#pragma unroll
          for (int ee = 0; ee < EC; ++ee) pj = ee == ie[j] ? ip[ee] : pj;
          s += pj;
          gw += ig[j] * iw[j];
        }
      }
#pragma unroll
      for (int j = 0; j < kTptMaxK; ++j) {
        if (j < k) {
          const float v = (ig[j] - gw) / s;
#pragma unroll
          for (int ee = 0; ee < EC; ++ee) dp[ee] += ee == ie[j] ? v : 0.f;
        }
      }
    }
    float c = 0.f;
#pragma unroll
    for (int e = 0; e < EC; ++e) c += ip[e] * dp[e];
    float dl[EC];
#pragma unroll
    for (int e = 0; e < EC; ++e) dl[e] = ip[e] * (dp[e] - c) * inv_tau;
    if (logits != nullptr) {  // z-loss term: lse of l / tau
      float m = -INFINITY, lt[EC];
#pragma unroll
      for (int e = 0; e < EC; ++e) {
        lt[e] = e < E ? ilt[e] * inv_tau : -INFINITY;
        m = fmaxf(m, lt[e]);
      }
      float se = 0.f;
#pragma unroll
      for (int e = 0; e < EC; ++e) se += e < E ? expf(lt[e] - m) : 0.f;
      const float lse = m + logf(se);
#pragma unroll
      for (int e = 0; e < EC; ++e) dl[e] += zc * lse * ip[e] * inv_tau;
    }
    if (E == EC) {
      float4* o = reinterpret_cast<float4*>(d_logits + t * EC);
#pragma unroll
      for (int i = 0; i < EC / 4; ++i) o[i] = make_float4(dl[4 * i], dl[4 * i + 1], dl[4 * i + 2], dl[4 * i + 3]);
    } else {
#pragma unroll
      for (int e = 0; e < EC; ++e)
        if (e < E) d_logits[t * E + e] = dl[e];
    }
    if (dlT != nullptr) {
#pragma unroll
      for (int e = 0; e < EC; ++e) {
        const float v = e < E ? dl[e] : 0.f;
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        dlT[static_cast<size_t>(e) * ldt + t] = h;
        dlT[static_cast<size_t>(EC + e) * ldt + t] = __float2bfloat16_rn(v - __bfloat162float(h));
      }
    }
    t += stride;
    if (t < T) load(t);
  }
}

template <typename T>
struct Io;
template <> struct Io<float> {
  static __device__ __forceinline__ float ld(const float* p) { return __ldg(p); }
  static __device__ __forceinline__ void st(float* p, float v) { *p = v; }
};
template <> struct Io<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void st(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};

// Vector access to CPT consecutive elements of a row (16-byte aligned for
// fp32 x 4, 8-byte for bf16 x 4; d is a multiple of 4, which the row stride
// and the column offsets keep).
template <typename T, int CPT>
struct Vec;
template <> struct Vec<float, 4> {
  static __device__ __forceinline__ void ld(const float* p, float (&v)[4]) {
    const float4 u = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  }
  static __device__ __forceinline__ void st(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};
template <> struct Vec<__nv_bfloat16, 4> {
  static __device__ __forceinline__ void ld(const __nv_bfloat16* p, float (&v)[4]) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    v[0] = __uint_as_float(u.x << 16); v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16); v[3] = __uint_as_float(u.y & 0xffff0000u);
  }
  static __device__ __forceinline__ void st(__nv_bfloat16* p, const float (&v)[4]) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<const uint32_t*>(&a),
                                              *reinterpret_cast<const uint32_t*>(&b));
  }
};
template <> struct Vec<float, 2> {
  static __device__ __forceinline__ void ld(const float* p, float (&v)[2]) {
    const float2 u = __ldg(reinterpret_cast<const float2*>(p));
    v[0] = u.x; v[1] = u.y;
  }
};
template <> struct Vec<__nv_bfloat16, 2> {
  static __device__ __forceinline__ void ld(const __nv_bfloat16* p, float (&v)[2]) {
    const uint32_t u = __ldg(reinterpret_cast<const unsigned int*>(p));
    v[0] = __uint_as_float(u << 16); v[1] = __uint_as_float(u & 0xffff0000u);
  }
};
template <typename T> struct Vec<T, 1> {
  static __device__ __forceinline__ void ld(const T* p, float (&v)[1]) { v[0] = Io<T>::ld(p); }
};

// dx[t, c] = sum_e dl[t, e] Wg[c, e], e in increasing order. Block: 128
// threads x 4 columns = 512 columns, 8 tiles of 16 tokens. Wg's columns are
// staged transposed per 16-expert chunk (once per block when E <= 16), so a
// thread reads its 4 columns in one conflict-free 16-byte load; each tile's
// dl rows are staged transposed (four 16-byte broadcasts per expert); Wg is
// read along its rows. With E > 16 every tile re-stages Wg, so a block then
// takes one tile (tiles = 1) and the grid is 8 times taller.
constexpr int kDxThreads = 128;
constexpr int kDxCols = 4 * kDxThreads;
constexpr int kDxTok = 16;
constexpr int kDxE = 16;
constexpr int kDxTiles = 8;

template <typename T>
__global__ void __launch_bounds__(kDxThreads)
bwd_dx(const float* __restrict__ dl, const T* __restrict__ wg, int Tn, int d, int E, int tiles,
       T* __restrict__ dx) {
  pdl_begin();
  __shared__ __align__(16) float wg_s[kDxE][kDxCols + 4];  // +4: the transposing stores spread over banks
  __shared__ __align__(16) float dl_s[kDxE][kDxTok];
  const int c = blockIdx.x * kDxCols + 4 * threadIdx.x;
  const bool one_chunk = E <= kDxE;
  auto stage_wg = [&](int e0, int ne) {
    for (int i = threadIdx.x; i < ne * kDxCols; i += kDxThreads) {
      const int cc = i / ne, e = i - cc * ne;
      const int col = blockIdx.x * kDxCols + cc;
      wg_s[e][cc] = col < d ? Io<T>::ld(wg + static_cast<size_t>(col) * E + e0 + e) : 0.f;
    }
  };
  if (one_chunk) stage_wg(0, E);  // read after the first tile's barrier
  for (int tile = 0; tile < tiles; ++tile) {
    const int t0 = (blockIdx.y * tiles + tile) * kDxTok;
    if (t0 >= Tn) break;  // the same for every thread of the block
    float acc[kDxTok][4];
#pragma unroll
    for (int i = 0; i < kDxTok; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int e0 = 0; e0 < E; e0 += kDxE) {
      const int ne = min(kDxE, E - e0);
      __syncthreads();  // the previous readers of the staged rows are done
      if (!one_chunk) stage_wg(e0, ne);
      for (int i = threadIdx.x; i < kDxE * kDxTok; i += kDxThreads) {
        const int tt = i / kDxE, e = i - tt * kDxE;
        const int t = t0 + tt;
        dl_s[e][tt] = (e < ne && t < Tn) ? __ldg(dl + static_cast<size_t>(t) * E + e0 + e) : 0.f;
      }
      __syncthreads();
      for (int e = 0; e < ne; ++e) {
        const float4 wv = *reinterpret_cast<const float4*>(&wg_s[e][4 * threadIdx.x]);
#pragma unroll
        for (int i = 0; i < kDxTok; i += 4) {
          const float4 g = *reinterpret_cast<const float4*>(&dl_s[e][i]);
          const float gi[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            acc[i + u][0] = fmaf(gi[u], wv.x, acc[i + u][0]);
            acc[i + u][1] = fmaf(gi[u], wv.y, acc[i + u][1]);
            acc[i + u][2] = fmaf(gi[u], wv.z, acc[i + u][2]);
            acc[i + u][3] = fmaf(gi[u], wv.w, acc[i + u][3]);
          }
        }
      }
    }
    if (c < d) {
#pragma unroll
      for (int i = 0; i < kDxTok; ++i)
        if (t0 + i < Tn) Vec<T, 4>::st(dx + static_cast<size_t>(t0 + i) * d + c, acc[i]);
    }
  }
}

// dWg partial of token split s: part[s][c][e] = sum over the split's tokens
// (increasing) of x[t, c] dl[t, e], for one EC-expert chunk (blockIdx.z;
// EC = 8, 16 or 32, the smallest that covers E up to 32). A thread owns
// CPT = 32 / EC consecutive columns (one vector load of x per token) and
// EC x CPT = 32 accumulators.
constexpr int kDwgThreads = 128;
constexpr int kDwgTok = 16;

template <typename T, int EC>
__global__ void __launch_bounds__(kDwgThreads)
bwd_dwg_part(const T* __restrict__ x, const float* __restrict__ dl, int Tn, int d, int E,
             int tok_per_split, float* __restrict__ part) {
  pdl_begin();
  constexpr int CPT = 32 / EC;
  __shared__ __align__(16) float dl_s[kDwgTok][EC];
  const int c = (blockIdx.x * kDwgThreads + threadIdx.x) * CPT;
  const int s = blockIdx.y, e0 = blockIdx.z * EC;
  const int ne = min(EC, E - e0);
  const int tb = s * tok_per_split, te = min(Tn, tb + tok_per_split);
  float acc[EC][CPT];
#pragma unroll
  for (int e = 0; e < EC; ++e)
#pragma unroll
    for (int j = 0; j < CPT; ++j) acc[e][j] = 0.f;
  for (int t0 = tb; t0 < te; t0 += kDwgTok) {
    __syncthreads();
    for (int i = threadIdx.x; i < kDwgTok * EC; i += kDwgThreads) {
      const int tt = i / EC, e = i - tt * EC;
      const int t = t0 + tt;
      dl_s[tt][e] = (e < ne && t < te) ? __ldg(dl + static_cast<size_t>(t) * E + e0 + e) : 0.f;
    }
    __syncthreads();
    float xv[kDwgTok][CPT];
#pragma unroll
    for (int i = 0; i < kDwgTok; ++i) {
      if (c < d && t0 + i < te) {
        Vec<T, CPT>::ld(x + static_cast<size_t>(t0 + i) * d + c, xv[i]);
      } else {
#pragma unroll
        for (int j = 0; j < CPT; ++j) xv[i][j] = 0.f;
      }
    }
#pragma unroll
    for (int i = 0; i < kDwgTok; ++i) {
#pragma unroll
      for (int e = 0; e < EC; e += 4) {
        const float4 g = *reinterpret_cast<const float4*>(&dl_s[i][e]);
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
          acc[e][j] = fmaf(xv[i][j], g.x, acc[e][j]);
          acc[e + 1][j] = fmaf(xv[i][j], g.y, acc[e + 1][j]);
          acc[e + 2][j] = fmaf(xv[i][j], g.z, acc[e + 2][j]);
          acc[e + 3][j] = fmaf(xv[i][j], g.w, acc[e + 3][j]);
        }
      }
    }
  }
  if (c < d) {
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      float* dst = part + (static_cast<size_t>(s) * d + c + j) * E + e0;
#pragma unroll
      for (int e = 0; e < EC; ++e)
        if (e < ne) dst[e] = acc[e][j];
    }
  }
}

// ------------------------------------------------ bf16, E <= 16: streaming
// ------------------------------------------------- tensor-core passes (bf16, E <= 16)
// The two T x d passes are contractions with a short side: dx = dL/dl Wg^T
// (K = E) and dWg = x^T dL/dl (K = T, N = E). On the tensor cores the bf16
// operands are exact; d_logits is fp32, so it enters as two bf16 terms,
// hi = bf16(v) and lo = bf16(v - hi), which together keep 16 bits of it
// (|v - hi - lo| <= 2^-17 |v| for |v| >= 2^-117, <= 2^-134 below); both
// products are summed in the fp32
// accumulator. EC is E rounded up to 8 or 16 (missing experts are zeros);
// the contraction has 2 EC terms per output: [hi | lo] against [W | W].
//
// 128-byte swizzle, K-major (the layout of a TMA SWIZZLE_128B box of
// 128-byte rows): the 16-byte chunk c of row r sits at
// (r / 8) * 1024 + (r % 8) * 128 + ((c ^ (r % 8)) * 16).
__device__ __forceinline__ uint8_t* sw128_chunk(uint8_t* base, int r, int c) {
  return base + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint32_t pack2_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// hi and lo bf16 terms of 8 fp32 values, packed 8 per 16-byte chunk.
__device__ __forceinline__ void split_hi_lo8(const float* v, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = v[2 * i], b = v[2 * i + 1];
    const float ah = __bfloat162float(__float2bfloat16_rn(a));
    const float bh = __bfloat162float(__float2bfloat16_rn(b));
    h[i] = pack2_bf16(ah, bh);
    l[i] = pack2_bf16(a - ah, b - bh);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// EC fp32 values of row t of a [T][E] array (zeros past E or T).
template <int EC>
__device__ __forceinline__ void load_row(const float* __restrict__ a, int t, int T, int E,
                                         float (&v)[EC]) {
  if (t < T && E == EC) {
    const float4* p = reinterpret_cast<const float4*>(a + static_cast<size_t>(t) * EC);
#pragma unroll
    for (int i = 0; i < EC / 4; ++i) {
      const float4 q = __ldg(p + i);
      v[4 * i] = q.x; v[4 * i + 1] = q.y; v[4 * i + 2] = q.z; v[4 * i + 3] = q.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < EC; ++e) v[e] = (t < T && e < E) ? __ldg(a + static_cast<size_t>(t) * E + e) : 0.f;
  }
}

// dx on the tensor cores: tile = 128 tokens x 256 columns, one MMA
// (M = 128, N = 256, K = 2 EC) per tile; A = [hi | lo] of the tile's d_logits
// rows, B = [Wg | Wg] of its columns, both written into shared memory by the
// block's threads (the block's 128 threads hold one token row each, loaded
// one tile ahead). The 4 warps then read their 32-row quarter of the fp32
// accumulator from tensor memory, round it to bf16, stage it per warp and
// store whole 128-byte row segments. Two blocks per SM (the dynamic shared
// memory is sized so that a third never fits: their accumulators take all
// 512 tensor-memory columns), so one block's MMA and operand writes overlap
// the other's stores. Tiles are numbered token tile major (u = tt * nct +
// ct) and the grid is a multiple of nct when it can be, so a block keeps one
// column tile and writes its B operand once. Waits are bounded.
constexpr int kDxTcThreads = 128;
constexpr int kDxTcTok = 128;
constexpr int kDxStageRow = 128 + 16;      // staged output row (16-byte pad: no bank conflicts)
constexpr int kDxStageWarp = 32 * kDxStageRow;
constexpr size_t kDxTcSmem = 86 * 1024;

// K = 2 EC is one 128-byte swizzle atom (EC <= 32) or two (EC = 64: hi in the
// first, lo in the second); a 64-expert tile is 128 columns wide so that two
// blocks still share an SM.
template <int EC>
struct DxTc {
  static constexpr int KB = (2 * EC + 63) / 64;        // K atoms
  static constexpr int TN = EC <= 32 ? 256 : 128;      // columns per tile (MMA N)
  static constexpr int A_ATOM = kDxTcTok * 128;        // 16 KB
  static constexpr int B_ATOM = TN * 128;
  static constexpr int A_BYTES = KB * A_ATOM;
  static constexpr int B_BYTES = KB * B_ATOM;
  static_assert(A_BYTES + B_BYTES + 4 * kDxStageWarp + 1024 <= static_cast<int>(kDxTcSmem), "dx smem");
};
static_assert(3 * (kDxTcSmem + 1024) > 228 * 1024, "at most two dx blocks per SM");

// Barrier over the 128 threads of a dx group (named barrier 1), and the same
// with an AND of a per-thread flag.
__device__ __forceinline__ void dx_group_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ int dx_group_and(int v) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.s32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, 128, q;\n\tselp.s32 %0, 1, 0, p;\n\t}"
      : "=r"(r) : "r"(v) : "memory");
  return r;
}

// The body of bwd_dx_tc, run by threads 0..127 of a block (block bid of nblk
// dx blocks; sm: the block's dynamic shared memory, 1024-aligned).
template <int EC>
__device__ __forceinline__ void dx_tc_body(const float* __restrict__ dl, const __nv_bfloat16* __restrict__ wg,
                                           int T, int d, int E, __nv_bfloat16* __restrict__ dx, Control* ctl,
                                           uint8_t* sm, int bid, int nblk) {
  static_assert(EC == 8 || EC == 16 || EC == 32 || EC == 64, "EC");
  using C = DxTc<EC>;
  constexpr int TN = C::TN;
  __shared__ __align__(8) uint64_t mma_bar;
  __shared__ uint32_t tmem_s;
  uint8_t* sa = sm;
  uint8_t* sb = sm + C::A_BYTES;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t* stg = sm + C::A_BYTES + C::B_BYTES + warp * kDxStageWarp;
  // 16-byte chunk c (8 K values) of row r of an operand of KB atoms
  auto chunk_a = [&](int r, int c) { return sw128_chunk(sa + (c >> 3) * C::A_ATOM, r, c & 7); };
  auto chunk_b = [&](int r, int c) { return sw128_chunk(sb + (c >> 3) * C::B_ATOM, r, c & 7); };
  if (tid == 0) {
    mbar_init(&mma_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_s, TN);
    tmem_relinquish();
  }
  tc_fence_before();
  dx_group_sync();
  tc_fence_after();
  const uint32_t tmem = tmem_s;
  const uint64_t limit = wait_limit_ns(ctl);
  const int ntt = (T + kDxTcTok - 1) / kDxTcTok, nct = (d + TN - 1) / TN;
  const int total = ntt * nct;
  constexpr uint32_t kIdesc = make_idesc_bf16(kDxTcTok, TN, true);
  float g[EC];
  if (bid < total) load_row<EC>(dl, (bid / nct) * kDxTcTok + tid, T, E, g);
  int cur_ct = -1;
  uint32_t phase = 0;
  bool pending = false;  // an MMA was issued and not yet waited for
  for (int u = bid; u < total; u += nblk) {
    const int tt = u / nct, ct = u - tt * nct;
    // A row tid: chunks [hi 0..EC) then [lo 0..EC), 8 values each
#pragma unroll
    for (int h = 0; h < EC / 8; ++h) {
      uint4 hi, lo;
      split_hi_lo8(g + 8 * h, hi, lo);
      *reinterpret_cast<uint4*>(chunk_a(tid, h)) = hi;
      *reinterpret_cast<uint4*>(chunk_a(tid, EC / 8 + h)) = lo;
    }
    if (ct != cur_ct) {
      // B rows = columns c of this tile: [Wg[c, 0..EC) | Wg[c, 0..EC)]
      for (int r = tid; r < TN; r += kDxTcThreads) {
        const int c = ct * TN + r;
        uint4 w[EC / 8];
        if (c < d && E == EC) {
          const uint4* p = reinterpret_cast<const uint4*>(wg + static_cast<size_t>(c) * EC);
#pragma unroll
          for (int h = 0; h < EC / 8; ++h) w[h] = __ldg(p + h);
        } else {
          uint16_t b[EC];
#pragma unroll
          for (int e = 0; e < EC; ++e)
            b[e] = (c < d && e < E) ? __bfloat16_as_ushort(wg[static_cast<size_t>(c) * E + e]) : 0;
#pragma unroll
          for (int h = 0; h < EC / 8; ++h)
            w[h] = make_uint4(b[8 * h] | (uint32_t(b[8 * h + 1]) << 16), b[8 * h + 2] | (uint32_t(b[8 * h + 3]) << 16),
                              b[8 * h + 4] | (uint32_t(b[8 * h + 5]) << 16), b[8 * h + 6] | (uint32_t(b[8 * h + 7]) << 16));
        }
#pragma unroll
        for (int h = 0; h < EC / 8; ++h) {
          *reinterpret_cast<uint4*>(chunk_b(r, h)) = w[h];
          *reinterpret_cast<uint4*>(chunk_b(r, EC / 8 + h)) = w[h];
        }
      }
      cur_ct = ct;
    }
    fence_proxy_async_smem();  // the generic-proxy writes above, before the MMA reads them
    tc_fence_before();
    dx_group_sync();
    tc_fence_after();
    if (tid == 0) {
      const uint32_t a_addr = smem_u32(sa), b_addr = smem_u32(sb);
#pragma unroll
      for (int kk = 0; kk < 2 * EC / 16; ++kk)
        umma_bf16(tmem, make_sw128_desc(a_addr + (kk >> 2) * C::A_ATOM + (kk & 3) * 32, 16, 1024),
                  make_sw128_desc(b_addr + (kk >> 2) * C::B_ATOM + (kk & 3) * 32, 16, 1024), kIdesc,
                  kk > 0 ? 1u : 0u);
      umma_commit(&mma_bar);
    }
    pending = true;
    // the next tile's d_logits rows are in flight during this tile's stores
    const int un = u + nblk;
    if (un < total) load_row<EC>(dl, (un / nct) * kDxTcTok + tid, T, E, g);
    int ok = 0;
    if (lane == 0) ok = mbar_wait_bounded(&mma_bar, phase, limit);
    ok = __shfl_sync(kFull, ok, 0);
    if (!dx_group_and(ok)) {
      if (tid == 0) set_error(ctl, MOE_DEVERR_TIMEOUT);
      break;
    }
    pending = false;
    phase ^= 1u;
    tc_fence_after();
    const long long t0 = static_cast<long long>(tt) * kDxTcTok + warp * 32;
    const int nrows = static_cast<int>(max(0LL, min(32LL, T - t0)));
    const int c0 = ct * TN;
    const int ncols = min(TN, d - c0);
    const uint32_t tq = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    if (nrows > 0) {
      for (int gc = 0; gc < ncols; gc += 64) {
        uint32_t v0[32], v1[32];
        tmem_ld_32x32b_x32(tq + gc, v0);
        tmem_ld_32x32b_x32(tq + gc + 32, v1);
        tmem_ld_wait();
        uint4* sp = reinterpret_cast<uint4*>(stg + lane * kDxStageRow);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          sp[i] = make_uint4(pack2_bf16(__uint_as_float(v0[8 * i]), __uint_as_float(v0[8 * i + 1])),
                             pack2_bf16(__uint_as_float(v0[8 * i + 2]), __uint_as_float(v0[8 * i + 3])),
                             pack2_bf16(__uint_as_float(v0[8 * i + 4]), __uint_as_float(v0[8 * i + 5])),
                             pack2_bf16(__uint_as_float(v0[8 * i + 6]), __uint_as_float(v0[8 * i + 7])));
          sp[4 + i] = make_uint4(pack2_bf16(__uint_as_float(v1[8 * i]), __uint_as_float(v1[8 * i + 1])),
                                 pack2_bf16(__uint_as_float(v1[8 * i + 2]), __uint_as_float(v1[8 * i + 3])),
                                 pack2_bf16(__uint_as_float(v1[8 * i + 4]), __uint_as_float(v1[8 * i + 5])),
                                 pack2_bf16(__uint_as_float(v1[8 * i + 6]), __uint_as_float(v1[8 * i + 7])));
        }
        __syncwarp();
        const int cq = lane & 7, rsub = lane >> 3;
        const bool col_ok = gc + cq * 8 < ncols;
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int rr = it * 4 + rsub;
          if (rr < nrows && col_ok)
            *reinterpret_cast<uint4*>(dx + static_cast<size_t>(t0 + rr) * d + c0 + gc + cq * 8) =
                *reinterpret_cast<const uint4*>(stg + rr * kDxStageRow + cq * 16);
        }
        __syncwarp();
      }
    }
    tc_fence_before();  // this tile's tensor-memory reads, before the next tile's barrier and MMA
  }
  if (pending && tid == 0) (void)mbar_wait_bounded(&mma_bar, phase, limit);
  tc_fence_before();
  dx_group_sync();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TN);
  }
}

template <int EC>
__global__ void __launch_bounds__(kDxTcThreads, 2)
bwd_dx_tc(const float* __restrict__ dl, const __nv_bfloat16* __restrict__ wg, int T, int d, int E,
          __nv_bfloat16* __restrict__ dx, Control* ctl) {
  pdl_begin();
  extern __shared__ uint8_t dx_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dx_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  dx_tc_body<EC>(dl, wg, T, d, E, dx, ctl, sm, blockIdx.x, gridDim.x);
}

// dWg on the tensor cores, per 128-column tile of x: D[c, n] = sum_t x[t, c]
// B[t, n] with A = x^T (M = 128 columns, MN-major: the rows of x as TMA
// loads them) and B = the bf16 terms of d_logits, [hi | lo] (N = 2 EC,
// K-major: the transposed copy dlT [2 EC][T] that bwd_logits_tpt writes). A unit
// is one 128-column tile x 64 tokens (16 KB of x); units are ordered tile by
// tile, tokens fastest, and every block takes the same number L of
// consecutive units (the last fewer), so all SMs stream equal shares of x.
// A block's units fall into one or more column tiles: per tile it sums its
// units in tensor memory and writes the fp32 sum (hi + lo terms added) as
// partial i of that tile, i = its rank among the tile's blocks. The last of
// a tile's blocks to finish (a ticket per tile and 32-column quarter, zeroed
// by bwd_logits_tpt) adds the tile's partials in order i = 0, 1, ... and writes
// d_wg: the result does not depend on which block finishes last.
//
// Warps: 0 TMA producer (x boxes and the dlT box per unit, 8-stage ring),
// 1 MMA issuer (4 MMAs of K = 16 per unit, double-buffered accumulator),
// 2..5 epilogue (tensor-memory lane quarter = warp % 4). Waits are bounded.
constexpr int kDwgTcThreads = 192;
constexpr int kDwgTcStages = 8;
constexpr int kMaxDwgStages = 8;
constexpr int kDwgTcCols = 128;
constexpr int kDwgTcTok = 64;
// Partials per column tile: enough for every SM to share one tile when d is
// small (2 x 160 SMs' worth), at least 32; the host keeps L large enough.
__host__ __device__ inline int dwg_max_contrib(int nct) { return max(32, (320 + nct - 1) / nct + 2); }

template <int EC>
struct DwgTc {
  static constexpr int N = 2 * EC;
  static constexpr int A_BYTES = kDwgTcCols * kDwgTcTok * 2;  // two 64-column boxes
  static constexpr int B_BYTES = N * kDwgTcTok * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;              // a multiple of 1024
  static constexpr int STAGES = EC <= 32 ? kDwgTcStages : 6;
  // beside a dx block (bwd_dxdwg_tc): what fits in kDxTcSmem
  static constexpr int FUSED_STAGES = EC <= 16 ? 4 : (EC == 32 ? 3 : 2);
  static constexpr int ACC = N < 32 ? 32 : N;                  // tensor-memory columns per accumulator
  static constexpr int TMEM = 2 * ACC;                         // a power of two >= 64
  static constexpr size_t SMEM = static_cast<size_t>(STAGES) * STAGE + 1024;
};

// The body of bwd_dwg_tc for block bid with an NST-stage ring, run by all
// kDwgTcThreads threads of a block (dwg_raw: its dynamic shared memory,
// before alignment).
template <int EC, int NST>
__device__ __forceinline__ void dwg_tc_body(const CUtensorMap* tmx_p, const CUtensorMap* tmg_p, int d,
                                            int E, int ntb, int total, int L, int maxc,
                                            float* __restrict__ part, int* __restrict__ tickets,
                                            float* __restrict__ d_wg, Control* ctl, uint8_t* dwg_raw,
                                            int bid) {
  using C = DwgTc<EC>;
  static_assert(C::STAGE % 1024 == 0, "stage alignment");
  static_assert(NST <= kMaxDwgStages, "ring barriers");
  __shared__ __align__(8) uint64_t full[kMaxDwgStages], empty[kMaxDwgStages];
  __shared__ __align__(8) uint64_t tfull[2], tempty[2], drain;
  __shared__ uint32_t tmem_s;
  __shared__ volatile int abort_s;
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dwg_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u0 = bid * L, u1 = min(total, u0 + L);
  const uint64_t limit = wait_limit_ns(ctl);
  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(&drain, 1);
    abort_s = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_s, C::TMEM);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_s;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(tmx_p);
      prefetch_tmap(tmg_p);
      int stage = 0;
      uint32_t phase = 0, issued_mask = 0, last_parity = 0;
      for (int u = u0; u < u1 && !abort_s; ++u) {
        const int j = u / ntb, tb = u - j * ntb;
        if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, limit)) {
          set_error(ctl, MOE_DEVERR_TIMEOUT);
          abort_s = 1;
          break;
        }
        uint8_t* sa = sm + stage * C::STAGE;
        mbar_arrive_expect_tx(&full[stage], C::STAGE);
        tma_load_2d(sa, tmx_p, &full[stage], j * kDwgTcCols, tb * kDwgTcTok);
        tma_load_2d(sa + C::A_BYTES / 2, tmx_p, &full[stage], j * kDwgTcCols + 64, tb * kDwgTcTok);
        tma_load_2d(sa + C::A_BYTES, tmg_p, &full[stage], tb * kDwgTcTok, 0);
        issued_mask |= 1u << stage;
        last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == NST) {
          stage = 0;
          phase ^= 1u;
        }
      }
      for (int s = 0; s < NST; ++s)
        if ((issued_mask >> s) & 1u)
          if (!mbar_wait_bounded(&full[s], (last_parity >> s) & 1u, limit)) set_error(ctl, MOE_DEVERR_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // A MN-major (bit 15), B K-major
      constexpr uint32_t kIdesc = make_idesc_bf16(kDwgTcCols, C::N, true) | (1u << 15);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool issued_any = false;
      int u = u0;
      while (u < u1 && !abort_s) {
        const int j = u / ntb;
        const int ue = min(u1, (j + 1) * ntb);
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, limit)) {
          set_error(ctl, MOE_DEVERR_TIMEOUT);
          abort_s = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * C::ACC;
        const int us = u;
        bool ok = true;
        for (; u < ue; ++u) {
          if (!mbar_wait_bounded(&full[stage], phase, limit)) {
            set_error(ctl, MOE_DEVERR_TIMEOUT);
            abort_s = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sm + stage * C::STAGE);
          const uint32_t b_addr = a_addr + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < kDwgTcTok / 16; ++kk)
            umma_bf16(d_tmem, make_sw128_desc(a_addr + kk * 2048, C::A_BYTES / 2, 1024),
                      make_sw128_desc(b_addr + kk * 32, 16, 1024), kIdesc,
                      (u != us || kk != 0) ? 1u : 0u);
          issued_any = true;
          umma_commit(&empty[stage]);
          if (++stage == NST) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (issued_any) {
        umma_commit(&drain);
        (void)mbar_wait_bounded(&drain, 0, limit);
      }
    }
  } else {
    // epilogue warps 2..5: columns 32 q .. 32 q + 31 of each tile
    const int q = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    int u = u0;
    while (u < u1) {
      const int j = u / ntb;
      const int ue = min(u1, (j + 1) * ntb);
      u = ue;
      int ok = 0;
      if (lane == 0) {
        ok = !abort_s && mbar_wait_bounded(&tfull[acc], acc_phase, limit);
        if (!ok && !abort_s) {
          set_error(ctl, MOE_DEVERR_TIMEOUT);
          abort_s = 1;
        }
      }
      if (!__shfl_sync(kFull, ok, 0)) break;
      tc_fence_after();
      float v[EC];
      {
        const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + acc * C::ACC;
        if constexpr (EC == 8) {
          uint32_t r[16];
          tmem_ld_32x32b_x16(ta, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(r[e]) + __uint_as_float(r[8 + e]);
        } else {
          // hi in columns [0, EC), lo in [EC, 2 EC), 16 at a time
#pragma unroll
          for (int h = 0; h < EC / 16; ++h) {
            uint32_t rh[16], rl[16];
            tmem_ld_32x32b_x16(ta + 16 * h, rh);
            tmem_ld_32x32b_x16(ta + EC + 16 * h, rl);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) v[16 * h + i] = __uint_as_float(rh[i]) + __uint_as_float(rl[i]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
      // this block's rank among the tile's blocks, and their number
      const int first = static_cast<int>((static_cast<long long>(j) * ntb) / L);
      const int last = static_cast<int>((static_cast<long long>(j + 1) * ntb - 1) / L);
      const int i = bid - first, n = last - first + 1;
      const int r = q * 32 + lane;
      float* mine = part + ((static_cast<size_t>(j) * maxc + i) * kDwgTcCols + r) * EC;
#pragma unroll
      for (int e = 0; e < EC; e += 4)
        *reinterpret_cast<float4*>(mine + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
      if (tickets == nullptr) continue;  // EC >= 32: bwd_dwg_tc_reduce adds the partials
      __threadfence();
      __syncwarp();
      int prev = 0;
      if (lane == 0) prev = atomicAdd(tickets + j * 4 + q, 1);
      prev = __shfl_sync(kFull, prev, 0);
      if (prev == n - 1) {
        __threadfence();
        const int c = j * kDwgTcCols + r;
        float sum[EC];
#pragma unroll
        for (int e = 0; e < EC; ++e) sum[e] = 0.f;
        // partials in batches whose loads are all in flight at once; added in order k
        constexpr int kBatch = EC <= 64 ? 64 / EC : 1;
        for (int k0 = 0; k0 < n; k0 += kBatch) {
          float4 t4[kBatch][EC / 4];
#pragma unroll
          for (int kb = 0; kb < kBatch; ++kb) {
            const float4* src = reinterpret_cast<const float4*>(
                part + ((static_cast<size_t>(j) * maxc + min(k0 + kb, n - 1)) * kDwgTcCols + r) * EC);
#pragma unroll
            for (int e4 = 0; e4 < EC / 4; ++e4) t4[kb][e4] = __ldcg(src + e4);
          }
#pragma unroll
          for (int kb = 0; kb < kBatch; ++kb) {
            if (k0 + kb < n) {
#pragma unroll
              for (int e4 = 0; e4 < EC / 4; ++e4) {
                sum[4 * e4] += t4[kb][e4].x;
                sum[4 * e4 + 1] += t4[kb][e4].y;
                sum[4 * e4 + 2] += t4[kb][e4].z;
                sum[4 * e4 + 3] += t4[kb][e4].w;
              }
            }
          }
        }
        if (c < d) {
#pragma unroll
          for (int e = 0; e < EC; ++e)
            if (e < E) d_wg[static_cast<size_t>(c) * E + e] = sum[e];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM);
  }
}

template <int EC>
__global__ void __launch_bounds__(kDwgTcThreads, 1)
bwd_dwg_tc(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmg, int d,
           int E, int ntb, int total, int L, int maxc, float* __restrict__ part,
           int* __restrict__ tickets, float* __restrict__ d_wg, Control* ctl) {
  pdl_begin();
  extern __shared__ uint8_t dwg_smem[];
  dwg_tc_body<EC, DwgTc<EC>::STAGES>(&tmx, &tmg, d, E, ntb, total, L, maxc, part, tickets, d_wg, ctl,
                                      dwg_smem, blockIdx.x);
}

// dx and dWg in one launch (bf16, both requested): blocks [0, ndwg) run the
// dWg body with a shorter ring (DwgTc<EC>::FUSED_STAGES), the rest the dx
// body on threads 0..127 (threads 128.. of those blocks have nothing to do).
// The shared memory (kDxTcSmem) and tensor memory (at most 384 columns) of
// one block of each kind fit one SM together, so every SM streams x for dWg
// and writes dx at the same time; at small T each pass alone is
// latency-bound.

template <int EC>
__global__ void __launch_bounds__(kDwgTcThreads, 2)
bwd_dxdwg_tc(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmg, int d,
             int E, int ntb, int total, int L, int maxc, float* __restrict__ part,
             int* __restrict__ tickets, float* __restrict__ d_wg, int ndwg,
             const float* __restrict__ dl, const __nv_bfloat16* __restrict__ wg, int T,
             __nv_bfloat16* __restrict__ dx, Control* ctl) {
  pdl_begin();
  static_assert(DwgTc<EC>::FUSED_STAGES * DwgTc<EC>::STAGE + 1024 <= static_cast<int>(kDxTcSmem), "fused smem");
  static_assert(DxTc<EC>::TN + DwgTc<EC>::TMEM <= 512, "fused tensor memory");
  extern __shared__ uint8_t both_smem[];
  if (static_cast<int>(blockIdx.x) < ndwg) {
    dwg_tc_body<EC, DwgTc<EC>::FUSED_STAGES>(&tmx, &tmg, d, E, ntb, total, L, maxc, part, tickets, d_wg, ctl,
                                     both_smem, blockIdx.x);
  } else if (threadIdx.x < kDxTcThreads) {
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(both_smem) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    dx_tc_body<EC>(dl, wg, T, d, E, dx, ctl, sm, static_cast<int>(blockIdx.x) - ndwg,
                   static_cast<int>(gridDim.x) - ndwg);
  }
}

// d_wg[c, e] = sum_s part[s][c][e], s increasing.
__global__ void __launch_bounds__(256)
bwd_dwg_reduce(const float* __restrict__ part, int nsplit, long long n, float* __restrict__ d_wg) {
  pdl_begin();
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float a = 0.f;
    for (int s = 0; s < nsplit; ++s) a += __ldg(part + static_cast<size_t>(s) * n + i);
    d_wg[i] = a;
  }
}

// Token splits of the dWg partials: at least 64 tokens each, at most 64, and
// at most 32 MB of partials (d * E * 4 bytes per split).
int dwg_splits(int T, int d, int E) {
  int s = (T + 63) / 64;
  const long long cap = (8LL << 20) / (static_cast<long long>(d) * E);
  if (s > 64) s = 64;
  if (s > cap) s = static_cast<int>(cap);
  return s < 1 ? 1 : s;
}

// The partials of bwd_dwg_tc for EC >= 32, where one block per tile adding
// about 150 / (d / 128) partials of 128 x EC floats would be a long serial
// tail: d_wg[c, e] = sum over the tile's blocks i = 0, 1, ... of
// part[tile][i][c % 128][e], a thread per 4 experts of a column (the same
// order as the in-kernel reduction: deterministic).
template <int EC>
__global__ void __launch_bounds__(256)
bwd_dwg_tc_reduce(const float* __restrict__ part, int d, int E, int ntb, int L, int maxc,
                  float* __restrict__ d_wg) {
  pdl_begin();
  const long long n = static_cast<long long>(d) * (EC / 4);
  for (long long i = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * 256) {
    const int c = static_cast<int>(i / (EC / 4)), e4 = static_cast<int>(i - static_cast<long long>(c) * (EC / 4));
    const int j = c / kDwgTcCols, r = c - j * kDwgTcCols;
    const int first = static_cast<int>((static_cast<long long>(j) * ntb) / L);
    const int last = static_cast<int>((static_cast<long long>(j + 1) * ntb - 1) / L);
    const float4* src = reinterpret_cast<const float4*>(part) +
                        ((static_cast<size_t>(j) * maxc) * kDwgTcCols + r) * (EC / 4) + e4;
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int k = 0; k < last - first + 1; ++k) {
      const float4 t4 = __ldg(src + static_cast<size_t>(k) * kDwgTcCols * (EC / 4));
      sum.x += t4.x;
      sum.y += t4.y;
      sum.z += t4.z;
      sum.w += t4.w;
    }
    const float v[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (4 * e4 + q < E) d_wg[static_cast<size_t>(c) * E + 4 * e4 + q] = v[q];
  }
}

// Tensor-core dWg (E <= 64): partials [column tile][dwg_max_contrib][128][EC],
// the transposed bf16 terms dlT [2 EC][ldt] and the tickets [column tile][4].
int dwg_tc_ec(int E) { return E <= 8 ? 8 : E <= 16 ? 16 : E <= 32 ? 32 : 64; }
long long dlt_ld(int T) { return (static_cast<long long>(T) + 15) / 16 * 16; }
int dwg_tc_tiles(int d) { return (d + kDwgTcCols - 1) / kDwgTcCols; }
size_t dwg_tc_part_bytes(int d, int E) {
  const int nct = dwg_tc_tiles(d);
  return static_cast<size_t>(nct) * dwg_max_contrib(nct) * kDwgTcCols * dwg_tc_ec(E) * 4;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

size_t route_backward_scratch_bytes(int T, int d, int E) {
  size_t part = static_cast<size_t>(dwg_splits(T, d, E)) * d * E * 4;
  size_t extra = 0;
  if (E <= 64) {
    part = std::max(part, dwg_tc_part_bytes(d, E));
    extra = align_up(static_cast<size_t>(2 * dwg_tc_ec(E)) * dlt_ld(T) * 2) +
            align_up(static_cast<size_t>(dwg_tc_tiles(d)) * 4 * 4) +
            align_up(static_cast<size_t>(kTptMaxBlocks) * 16 * 4);
  }
  return align_up(static_cast<size_t>(E) * 4) + align_up(static_cast<size_t>(T) * E * 4) + align_up(part) +
         extra + align_up(static_cast<size_t>(kHistMaxBlocks) * E * 4);
}

cudaError_t launch_route_backward(const void* x, const void* wg, moe_dtype_t dt, int T, int d,
                                  int E, int k, const float* probs, const float* logits,
                                  const int32_t* idx, const float* w, const float* d_w,
                                  float d_aux, float d_z, float temperature, float* d_logits,
                                  void* dx, float* d_wg, void* scratch, Control* ctl,
                                  cudaStream_t s) {
  uint8_t* sc = static_cast<uint8_t*>(scratch);
  int32_t* counts = reinterpret_cast<int32_t*>(sc);
  sc += align_up(static_cast<size_t>(E) * 4);
  float* dl = d_logits != nullptr ? d_logits : reinterpret_cast<float*>(sc);
  sc += align_up(static_cast<size_t>(T) * E * 4);
  float* part = reinterpret_cast<float*>(sc);
  size_t part_bytes = static_cast<size_t>(dwg_splits(T, d, E)) * d * E * 4;
  if (E <= 64) part_bytes = std::max(part_bytes, dwg_tc_part_bytes(d, E));
  sc += align_up(part_bytes);
  __nv_bfloat16* dlT = nullptr;
  int* tickets = nullptr;
  int32_t* hist_part = nullptr;
  if (E <= 64) {
    dlT = reinterpret_cast<__nv_bfloat16*>(sc);
    sc += align_up(static_cast<size_t>(2 * dwg_tc_ec(E)) * dlt_ld(T) * 2);
    tickets = reinterpret_cast<int*>(sc);
    sc += align_up(static_cast<size_t>(dwg_tc_tiles(d)) * 4 * 4);
    hist_part = reinterpret_cast<int32_t*>(sc);
    sc += align_up(static_cast<size_t>(kTptMaxBlocks) * 16 * 4);
  }
  int32_t* hist_blocks = reinterpret_cast<int32_t*>(sc);  // the last region
  const float inv_tau = 1.0f / temperature;
  const bool aux = d_aux != 0.0f;
  // at most 16 experts and many picks: d_logits with a thread per token
  // (rows read and written as 16-byte vectors when E is 8 or 16); bf16 with
  // at most 64 experts: both T x d passes on the tensor cores
  const bool tpt = E <= 16 && k <= kTptMaxK && static_cast<long long>(T) * k >= kTptMinPicks &&
                   aligned16(probs) && aligned16(dl) && (d_z == 0.0f || aligned16(logits));
  const bool tc = E <= 64 && dt == MOE_BF16 && d % 8 == 0 && T > 0 && aligned16(x) && aligned16(wg) &&
                  aligned16(dl);
  const int ec = dwg_tc_ec(E);
  const bool tc_dwg = tc && d_wg != nullptr;
  cudaError_t err = cudaSuccess;
  if (T > 0 && tpt) {
    // large T: thread per token, the pick counts in the same launch
    // (cooperative: at most as many blocks as are resident)
    auto kern = E <= 8 ? bwd_logits_tpt<8> : bwd_logits_tpt<16>;
    int g = std::min((T + kTptThreads - 1) / kTptThreads, kTptMaxBlocks);
    if (aux) {
      int per_sm = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kTptThreads, 0) != cudaSuccess ||
          per_sm < 1)
        return cudaErrorInvalidConfiguration;
      g = std::min(g, per_sm * num_sms());
    }
    err = launch_pdl(kern, dim3(g), dim3(kTptThreads), 0, s, aux, probs, d_z != 0.0f ? logits : nullptr,
                     idx, w, d_w, aux ? 1 : 0, hist_part, d_aux, d_z, inv_tau, T, E, k, dl,
                     tc_dwg ? dlT : nullptr, static_cast<int>(dlt_ld(T)), tc_dwg && ec <= 16 ? tickets : nullptr,
                     dwg_tc_tiles(d) * 4, ctl);
    if (err != cudaSuccess) return err;
  } else if (T > 0) {
    if (aux) {
      const long long S = static_cast<long long>(T) * k, S4 = S / 4;
      const int hb = S <= kHistOneBlock ? 1 : static_cast<int>(std::max<long long>(
          1, std::min<long long>(kHistMaxBlocks, (S4 + kHistThreads - 1) / kHistThreads)));
      const long long per4 = (S4 + hb - 1) / hb;
      err = launch_pdl(bwd_hist, dim3(hb), dim3(kHistThreads), 0, s, false, idx, S, E, per4, hist_blocks,
                       counts, ctl);
      if (err != cudaSuccess) return err;
    }
    const int epl = (E + 31) / 32;
    auto kern = epl <= 1 ? bwd_logits<1> : epl <= 2 ? bwd_logits<2> : epl <= 4 ? bwd_logits<4>
                                                                              : bwd_logits<8>;
    const int grid = std::max(1, std::min((T + kLogitWarps - 1) / kLogitWarps, 4 * num_sms()));
    err = launch_pdl(kern, dim3(grid), dim3(kLogitWarps * 32), 0, s, false, probs,
                     d_z != 0.0f ? logits : nullptr, idx, w, d_w, aux ? counts : nullptr, d_aux,
                     d_z, inv_tau, T, E, k, dl, tc_dwg ? dlT : nullptr, ec, static_cast<int>(dlt_ld(T)),
                     tc_dwg && ec <= 16 ? tickets : nullptr, dwg_tc_tiles(d) * 4, ctl);
    if (err != cudaSuccess) return err;
  }
  // both passes requested, EC <= 16: one launch runs them side by side (for
  // EC = 64 the 2-stage dWg ring that fits beside a dx block measured slower
  // than the two launches: 70.8 against 63.5 us on the capacity workload)
  const bool fuse = tc && dx != nullptr && d_wg != nullptr && ec <= 16;
  if (T > 0 && !fuse) {
    if (dx != nullptr && tc) {
      const int tn = ec <= 32 ? DxTc<8>::TN : DxTc<64>::TN;
      const int nct = (d + tn - 1) / tn;
      const int tiles = ((T + kDxTcTok - 1) / kDxTcTok) * nct;
      const int slots = 2 * num_sms();
      const int g = std::min(tiles, nct <= slots ? slots / nct * nct : slots);
      auto kern = ec == 8 ? bwd_dx_tc<8> : ec == 16 ? bwd_dx_tc<16> : ec == 32 ? bwd_dx_tc<32> : bwd_dx_tc<64>;
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kDxTcSmem));
      err = launch_pdl(kern, dim3(g), dim3(kDxTcThreads), kDxTcSmem, s, false,
                       static_cast<const float*>(dl), static_cast<const __nv_bfloat16*>(wg), T, d, E,
                       static_cast<__nv_bfloat16*>(dx), ctl);
      if (err != cudaSuccess) return err;
    } else if (dx != nullptr) {
      const int tiles = E <= kDxE ? kDxTiles : 1;
      const dim3 g((d + kDxCols - 1) / kDxCols, (T + kDxTok * tiles - 1) / (kDxTok * tiles));
      err = dt == MOE_BF16
                ? launch_pdl(bwd_dx<__nv_bfloat16>, g, dim3(kDxThreads), 0, s, false, dl,
                             static_cast<const __nv_bfloat16*>(wg), T, d, E, tiles,
                             static_cast<__nv_bfloat16*>(dx))
                : launch_pdl(bwd_dx<float>, g, dim3(kDxThreads), 0, s, false, dl,
                             static_cast<const float*>(wg), T, d, E, tiles, static_cast<float*>(dx));
      if (err != cudaSuccess) return err;
    }
  }
  if (tc_dwg) {
    // equal shares of 64-token x 128-column units; L keeps a tile's blocks <= maxc
    // (with the fused launch: of one block per SM beside the dx blocks)
    const int ntb = (T + kDwgTcTok - 1) / kDwgTcTok;
    const int nct = dwg_tc_tiles(d);
    const int maxc = dwg_max_contrib(nct);
    const long long total = static_cast<long long>(ntb) * nct;
    if (total > 0x7fffffffLL) return cudaErrorInvalidValue;
    long long L = (total + num_sms() - 1) / num_sms();
    L = std::max<long long>(L, (ntb + maxc - 2) / (maxc - 1));
    const int G = static_cast<int>((total + L - 1) / L);
    CUtensorMap tmx, tmg;
    if (!make_tma_2d_bf16(&tmx, x, static_cast<uint64_t>(T), static_cast<uint64_t>(d), kDwgTcTok) ||
        !make_tma_2d_bf16_ld(&tmg, dlT, static_cast<uint64_t>(2 * ec), static_cast<uint64_t>(T),
                             static_cast<uint64_t>(dlt_ld(T)), static_cast<uint32_t>(2 * ec)))
      return cudaErrorInvalidValue;
    auto launch_reduce = [&]() -> cudaError_t {
      const long long nout = static_cast<long long>(d) * (ec / 4);
      const int rg = static_cast<int>(std::min<long long>((nout + 255) / 256, 8LL * num_sms()));
      auto red = ec == 32 ? bwd_dwg_tc_reduce<32> : bwd_dwg_tc_reduce<64>;
      return launch_pdl(red, dim3(std::max(rg, 1)), dim3(256), 0, s, false, static_cast<const float*>(part), d, E,
                        ntb, static_cast<int>(L), maxc, d_wg);
    };
    if (fuse) {
      const int tn = ec <= 32 ? DxTc<8>::TN : DxTc<64>::TN;
      const int nct_x = (d + tn - 1) / tn;
      const int tiles = ((T + kDxTcTok - 1) / kDxTcTok) * nct_x;
      const int sms = num_sms();
      const int gx = std::max(1, std::min(tiles, nct_x <= sms ? sms / nct_x * nct_x : sms));
      auto kf = ec == 8 ? bwd_dxdwg_tc<8> : ec == 16 ? bwd_dxdwg_tc<16> : ec == 32 ? bwd_dxdwg_tc<32> : bwd_dxdwg_tc<64>;
      cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kDxTcSmem));
      err = launch_pdl(kf, dim3(G + gx), dim3(kDwgTcThreads), kDxTcSmem, s, false, tmx, tmg, d, E, ntb,
                       static_cast<int>(total), static_cast<int>(L), maxc, part, ec <= 16 ? tickets : nullptr,
                       d_wg, G, static_cast<const float*>(dl), static_cast<const __nv_bfloat16*>(wg), T,
                       static_cast<__nv_bfloat16*>(dx), ctl);
      if (err != cudaSuccess || ec <= 16) return err;
      return launch_reduce();
    }
    const size_t smem = ec == 8 ? DwgTc<8>::SMEM : ec == 16 ? DwgTc<16>::SMEM
                      : ec == 32 ? DwgTc<32>::SMEM : DwgTc<64>::SMEM;
    auto kern = ec == 8 ? bwd_dwg_tc<8> : ec == 16 ? bwd_dwg_tc<16> : ec == 32 ? bwd_dwg_tc<32> : bwd_dwg_tc<64>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    err = launch_pdl(kern, dim3(G), dim3(kDwgTcThreads), smem, s, false, tmx, tmg, d, E, ntb,
                     static_cast<int>(total), static_cast<int>(L), maxc, part,
                     ec <= 16 ? tickets : nullptr, d_wg, ctl);
    if (err != cudaSuccess || ec <= 16) return err;
    err = launch_reduce();
  } else if (d_wg != nullptr) {
    const int ns = dwg_splits(T, d, E);
    const int tps = T > 0 ? (T + ns - 1) / ns : 0;
    const int ec = E <= 8 ? 8 : (E <= 16 ? 16 : 32);
    const int cols = kDwgThreads * (32 / ec);  // columns per block
    const dim3 g((d + cols - 1) / cols, ns, (E + ec - 1) / ec);
    if (dt == MOE_BF16) {
      const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
      err = ec == 8    ? launch_pdl(bwd_dwg_part<__nv_bfloat16, 8>, g, dim3(kDwgThreads), 0, s, false, xb,
                                    static_cast<const float*>(dl), T, d, E, tps, part)
            : ec == 16 ? launch_pdl(bwd_dwg_part<__nv_bfloat16, 16>, g, dim3(kDwgThreads), 0, s, false, xb,
                                    static_cast<const float*>(dl), T, d, E, tps, part)
                       : launch_pdl(bwd_dwg_part<__nv_bfloat16, 32>, g, dim3(kDwgThreads), 0, s, false, xb,
                                    static_cast<const float*>(dl), T, d, E, tps, part);
    } else {
      const float* xf = static_cast<const float*>(x);
      err = ec == 8    ? launch_pdl(bwd_dwg_part<float, 8>, g, dim3(kDwgThreads), 0, s, false, xf,
                                    static_cast<const float*>(dl), T, d, E, tps, part)
            : ec == 16 ? launch_pdl(bwd_dwg_part<float, 16>, g, dim3(kDwgThreads), 0, s, false, xf,
                                    static_cast<const float*>(dl), T, d, E, tps, part)
                       : launch_pdl(bwd_dwg_part<float, 32>, g, dim3(kDwgThreads), 0, s, false, xf,
                                    static_cast<const float*>(dl), T, d, E, tps, part);
    }
    if (err != cudaSuccess) return err;
    const long long n = static_cast<long long>(d) * E;
    const int rg = static_cast<int>(std::min<long long>((n + 255) / 256, 8LL * num_sms()));
    err = launch_pdl(bwd_dwg_reduce, dim3(std::max(rg, 1)), dim3(256), 0, s, false,
                     static_cast<const float*>(part), ns, n, d_wg);
  }
  return err;
}

}  // namespace moe
