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
  auto add = [&](int e) {
    if (e < 0 || e >= E) set_error(ctl, MOE_DEVERR_EXPERT_RANGE);
    else atomicAdd(&h[e], 1);
  };
  // four picks per 16-byte load (idx is 16-byte aligned), then the tail
  const long long S4 = S / 4;
  for (long long q = threadIdx.x; q < S4; q += blockDim.x) {
    const int4 v = __ldg(reinterpret_cast<const int4*>(idx) + q);
    add(v.x);
    add(v.y);
    add(v.z);
    add(v.w);
  }
  for (long long s = S4 * 4 + threadIdx.x; s < S; s += blockDim.x) add(__ldg(idx + s));
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

}  // namespace

size_t route_backward_scratch_bytes(int T, int d, int E) {
  return align_up(static_cast<size_t>(E) * 4) + align_up(static_cast<size_t>(T) * E * 4) +
         align_up(static_cast<size_t>(dwg_splits(T, d, E)) * d * E * 4);
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
  if (d_wg != nullptr) {
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
