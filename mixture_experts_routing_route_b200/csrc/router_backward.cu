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
// Kernels: an expert histogram of the picks (f, when d_aux != 0), d_logits
// with a warp per token, dx with a column per thread over 32-token tiles, and
// dWg as per-token-split partials added in split order (deterministic).
// fp32 arithmetic throughout; dx is rounded once to the input dtype.
#include "common.cuh"

#include <cmath>

namespace moe {
namespace {

constexpr unsigned kFull = 0xffffffffu;

// One block: counts[e] = slots that picked expert e (before any drop).
__global__ void __launch_bounds__(1024)
bwd_hist(const int32_t* __restrict__ idx, long long S, int E, int32_t* __restrict__ counts,
         Control* ctl) {
  pdl_begin();
  __shared__ int h[256];  // E <= 256
  for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
  __syncthreads();
  for (long long s = threadIdx.x; s < S; s += blockDim.x) {
    const int e = __ldg(idx + s);
    if (e < 0 || e >= E) {
      set_error(ctl, MOE_DEVERR_EXPERT_RANGE);
      continue;
    }
    atomicAdd(&h[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) counts[e] = h[e];
}

constexpr int kLogitWarps = 8;

// Warp per token; lane holds experts lane + 32 q, q < EPL.
template <int EPL>
__global__ void __launch_bounds__(kLogitWarps * 32)
bwd_logits(const float* __restrict__ probs, const float* __restrict__ logits,
           const int32_t* __restrict__ idx, const float* __restrict__ w,
           const float* __restrict__ d_w, const int32_t* __restrict__ counts, float d_aux,
           float d_z, float inv_tau, int T, int E, int k, float* __restrict__ d_logits,
           Control* ctl) {
  pdl_begin();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
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
  for (int t = blockIdx.x * kLogitWarps + warp; t < T; t += gridDim.x * kLogitWarps) {
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

constexpr int kCols = 256;   // columns of d per block (a thread each)
constexpr int kTok = 32;     // tokens per tile
constexpr int kEChunk = 32;  // experts staged at a time

// dx[t, c] = sum_e dl[t, e] Wg[c, e], e in increasing order. Block: 256
// columns x 32 tokens; Wg's columns and dl's rows are staged per 32-expert
// chunk, transposed so that a thread reads its column (conflict-free) and a
// token quadruple (one 16-byte broadcast).
template <typename T>
__global__ void __launch_bounds__(kCols, 2)
bwd_dx(const float* __restrict__ dl, const T* __restrict__ wg, int Tn, int d, int E,
       T* __restrict__ dx) {
  pdl_begin();
  __shared__ float wg_s[kEChunk][kCols];
  __shared__ __align__(16) float dl_s[kEChunk][kTok];
  const int c = blockIdx.x * kCols + threadIdx.x;
  const int t0 = blockIdx.y * kTok;
  float acc[kTok];
#pragma unroll
  for (int i = 0; i < kTok; ++i) acc[i] = 0.f;
  for (int e0 = 0; e0 < E; e0 += kEChunk) {
    const int ne = min(kEChunk, E - e0);
    __syncthreads();
    for (int i = threadIdx.x; i < kEChunk * kCols; i += kCols) {
      const int e = i / kCols, cc = i - e * kCols;
      const int col = blockIdx.x * kCols + cc;
      wg_s[e][cc] = (e < ne && col < d) ? Io<T>::ld(wg + static_cast<size_t>(col) * E + e0 + e) : 0.f;
    }
    for (int i = threadIdx.x; i < kEChunk * kTok; i += kCols) {
      const int tt = i / kEChunk, e = i - tt * kEChunk;
      const int t = t0 + tt;
      dl_s[e][tt] = (e < ne && t < Tn) ? __ldg(dl + static_cast<size_t>(t) * E + e0 + e) : 0.f;
    }
    __syncthreads();
    for (int e = 0; e < ne; ++e) {
      const float wv = wg_s[e][threadIdx.x];
#pragma unroll
      for (int i = 0; i < kTok; i += 4) {
        const float4 g = *reinterpret_cast<const float4*>(&dl_s[e][i]);
        acc[i] = fmaf(g.x, wv, acc[i]);
        acc[i + 1] = fmaf(g.y, wv, acc[i + 1]);
        acc[i + 2] = fmaf(g.z, wv, acc[i + 2]);
        acc[i + 3] = fmaf(g.w, wv, acc[i + 3]);
      }
    }
  }
  if (c < d) {
#pragma unroll
    for (int i = 0; i < kTok; ++i)
      if (t0 + i < Tn) Io<T>::st(dx + static_cast<size_t>(t0 + i) * d + c, acc[i]);
  }
}

// dWg partial of token split s: part[s][c][e] = sum over the split's tokens
// (increasing) of x[t, c] dl[t, e], for one 32-expert chunk (blockIdx.z).
template <typename T>
__global__ void __launch_bounds__(kCols)
bwd_dwg_part(const T* __restrict__ x, const float* __restrict__ dl, int Tn, int d, int E,
             int tok_per_split, float* __restrict__ part) {
  pdl_begin();
  __shared__ __align__(16) float dl_s[kTok][kEChunk];
  const int c = blockIdx.x * kCols + threadIdx.x;
  const int s = blockIdx.y, e0 = blockIdx.z * kEChunk;
  const int ne = min(kEChunk, E - e0);
  const int tb = s * tok_per_split, te = min(Tn, tb + tok_per_split);
  float acc[kEChunk];
#pragma unroll
  for (int i = 0; i < kEChunk; ++i) acc[i] = 0.f;
  for (int t0 = tb; t0 < te; t0 += kTok) {
    __syncthreads();
    for (int i = threadIdx.x; i < kTok * kEChunk; i += kCols) {
      const int tt = i / kEChunk, e = i - tt * kEChunk;
      const int t = t0 + tt;
      dl_s[tt][e] = (e < ne && t < te) ? __ldg(dl + static_cast<size_t>(t) * E + e0 + e) : 0.f;
    }
    __syncthreads();
    float xv[kTok];
#pragma unroll
    for (int i = 0; i < kTok; ++i)
      xv[i] = (c < d && t0 + i < te) ? Io<T>::ld(x + static_cast<size_t>(t0 + i) * d + c) : 0.f;
#pragma unroll
    for (int i = 0; i < kTok; ++i) {
#pragma unroll
      for (int e = 0; e < kEChunk; e += 4) {
        const float4 g = *reinterpret_cast<const float4*>(&dl_s[i][e]);
        acc[e] = fmaf(xv[i], g.x, acc[e]);
        acc[e + 1] = fmaf(xv[i], g.y, acc[e + 1]);
        acc[e + 2] = fmaf(xv[i], g.z, acc[e + 2]);
        acc[e + 3] = fmaf(xv[i], g.w, acc[e + 3]);
      }
    }
  }
  if (c < d) {
    float* dst = part + (static_cast<size_t>(s) * d + c) * E + e0;
#pragma unroll
    for (int e = 0; e < kEChunk; ++e)
      if (e < ne) dst[e] = acc[e];
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

int dwg_splits(int T) {
  const int s = (T + 127) / 128;  // about 128 tokens per split
  return s < 1 ? 1 : (s > 32 ? 32 : s);
}

}  // namespace

size_t route_backward_scratch_bytes(int T, int d, int E) {
  return align_up(static_cast<size_t>(E) * 4) + align_up(static_cast<size_t>(T) * E * 4) +
         align_up(static_cast<size_t>(dwg_splits(T)) * d * E * 4);
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
  const float inv_tau = 1.0f / temperature;
  const bool aux = d_aux != 0.0f;
  cudaError_t err = cudaSuccess;
  if (T > 0) {
    if (aux) {
      err = launch_pdl(bwd_hist, dim3(1), dim3(1024), 0, s, false, idx, static_cast<long long>(T) * k,
                       E, counts, ctl);
      if (err != cudaSuccess) return err;
    }
    const int epl = (E + 31) / 32;
    auto kern = epl <= 1 ? bwd_logits<1> : epl <= 2 ? bwd_logits<2> : epl <= 4 ? bwd_logits<4>
                                                                              : bwd_logits<8>;
    const int grid = std::max(1, std::min((T + kLogitWarps - 1) / kLogitWarps, 8 * num_sms()));
    err = launch_pdl(kern, dim3(grid), dim3(kLogitWarps * 32), 0, s, false, probs,
                     d_z != 0.0f ? logits : nullptr, idx, w, d_w, aux ? counts : nullptr, d_aux,
                     d_z, inv_tau, T, E, k, dl, ctl);
    if (err != cudaSuccess) return err;
    if (dx != nullptr) {
      const dim3 g((d + kCols - 1) / kCols, (T + kTok - 1) / kTok);
      err = dt == MOE_BF16
                ? launch_pdl(bwd_dx<__nv_bfloat16>, g, dim3(kCols), 0, s, false, dl,
                             static_cast<const __nv_bfloat16*>(wg), T, d, E, static_cast<__nv_bfloat16*>(dx))
                : launch_pdl(bwd_dx<float>, g, dim3(kCols), 0, s, false, dl,
                             static_cast<const float*>(wg), T, d, E, static_cast<float*>(dx));
      if (err != cudaSuccess) return err;
    }
  }
  if (d_wg != nullptr) {
    const int ns = dwg_splits(T);
    const int tps = T > 0 ? (T + ns - 1) / ns : 0;
    const dim3 g((d + kCols - 1) / kCols, ns, (E + kEChunk - 1) / kEChunk);
    err = dt == MOE_BF16
              ? launch_pdl(bwd_dwg_part<__nv_bfloat16>, g, dim3(kCols), 0, s, false,
                           static_cast<const __nv_bfloat16*>(x), static_cast<const float*>(dl), T, d, E,
                           tps, part)
              : launch_pdl(bwd_dwg_part<float>, g, dim3(kCols), 0, s, false,
                           static_cast<const float*>(x), static_cast<const float*>(dl), T, d, E, tps,
                           part);
    if (err != cudaSuccess) return err;
    const long long n = static_cast<long long>(d) * E;
    const int rg = static_cast<int>(std::min<long long>((n + 255) / 256, 8LL * num_sms()));
    err = launch_pdl(bwd_dwg_reduce, dim3(std::max(rg, 1)), dim3(256), 0, s, false,
                     static_cast<const float*>(part), ns, n, d_wg);
  }
  return err;
}

}  // namespace moe
