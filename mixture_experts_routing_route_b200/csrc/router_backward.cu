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
#include "ptx.cuh"

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

// ------------------------------------------------ bf16, E <= 16: streaming
// The two T x d passes of the Mixtral-sized router are pure streams (E
// multiply-adds per element): dx writes T x d, dWg reads x once. These
// kernels give each thread 8 consecutive columns (one 16-byte bf16 vector
// per token row) so that every row of x or dx is touched by whole 16-byte
// accesses, keep the per-column Wg values or accumulators in registers, and
// stage each block's d_logits tile in shared memory once.
constexpr int kFastThreads = 128;   // dx: 128 x 8 = 1024 columns per block
constexpr int kFastTok = 32;        // dx: tokens per block
constexpr int kFastDwgThreads = 128;  // dWg: 128 x 8 = 1024 columns per block

__device__ __forceinline__ void bf16x8_to_f32(const uint4 u, float (&v)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint4 f32x8_to_bf16(const float (&v)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// dx[t, c] = sum_e dl[t, e] Wg[c, e], e in increasing order (the order of
// bwd_dx). EC >= E (8 or 16); d a multiple of 8. The block's Wg rows
// [c0, c0 + 1024) are one contiguous range of memory: they are copied to
// shared memory with 16-byte loads, then each thread keeps its 8 rows in
// registers; the block's d_logits rows are staged once.
template <int EC>
__global__ void __launch_bounds__(kFastThreads)
bwd_dx_fast(const float* __restrict__ dl, const __nv_bfloat16* __restrict__ wg, int Tn, int d, int E,
            __nv_bfloat16* __restrict__ dx) {
  pdl_begin();
  extern __shared__ __align__(16) uint8_t dx_sm[];
  __nv_bfloat16* wg_s = reinterpret_cast<__nv_bfloat16*>(dx_sm);                       // [2048][E]
  float* dl_s = reinterpret_cast<float*>(dx_sm + kFastThreads * 8 * EC * 2);           // [kFastTok][EC]
  const int c0 = blockIdx.x * kFastThreads * 8;
  const int ncol = min(kFastThreads * 8, d - c0);
  const int c = c0 + threadIdx.x * 8;
  const int t0 = blockIdx.y * kFastTok;
  {
    const long long n16 = static_cast<long long>(ncol) * E * 2 / 16;  // a whole number: ncol % 8 == 0
    const uint4* src = reinterpret_cast<const uint4*>(wg + static_cast<size_t>(c0) * E);
    for (long long i = threadIdx.x; i < n16; i += kFastThreads)
      reinterpret_cast<uint4*>(wg_s)[i] = __ldg(src + i);
  }
  for (int i = threadIdx.x; i < kFastTok * EC; i += kFastThreads) {
    const int tt = i / EC, e = i - tt * EC;
    const int t = t0 + tt;
    dl_s[i] = (e < E && t < Tn) ? __ldg(dl + static_cast<size_t>(t) * E + e) : 0.f;
  }
  __syncthreads();
  if (c >= d) return;
  float wv[8][EC];
#pragma unroll
  for (int jj = 0; jj < 8; ++jj)
#pragma unroll
    for (int e = 0; e < EC; ++e)
      wv[jj][e] = e < E ? __bfloat162float(wg_s[(threadIdx.x * 8 + jj) * E + e]) : 0.f;
  const int nt = min(kFastTok, Tn - t0);
#pragma unroll 4
  for (int tt = 0; tt < nt; ++tt) {
    float acc[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) acc[jj] = 0.f;
#pragma unroll
    for (int e4 = 0; e4 < EC; e4 += 4) {
      const float4 g4 = *reinterpret_cast<const float4*>(dl_s + tt * EC + e4);
      const float g[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) acc[jj] = fmaf(g[q], wv[jj][e4 + q], acc[jj]);
    }
    *reinterpret_cast<uint4*>(dx + static_cast<size_t>(t0 + tt) * d + c) = f32x8_to_bf16(acc);
  }
}

size_t dx_fast_smem(int ec) {
  return static_cast<size_t>(kFastThreads) * 8 * ec * 2 + static_cast<size_t>(kFastTok) * ec * 4;
}

// dWg partial of token split s: part[s][c][e] = sum over the split's tokens
// (increasing) of x[t, c] dl[t, e]. EC >= E (8 or 16); d a multiple of 8.
// Block = G row groups of 128 threads, one block per SM; a group's thread
// owns 8 columns of the block's 1024 (G = 4 for EC = 8, 2 for EC = 16, so
// that the accumulators fit). Thread 0 streams the split's rows of that
// column slice (2 KB per token row) with bulk copies into a 4-stage ring of
// 16 rows (128 KB in flight per SM, the copy engine's, not registers); group
// g adds rows g, g + G, ... of each stage. At the end groups 1..G-1 leave
// their sums in the idle ring and group 0 adds them in group order.
// Waits are bounded.
constexpr int kDwgBulkStages = 4;
constexpr int kDwgBulkRows = 16;
constexpr int kDwgBulkRowBytes = kFastDwgThreads * 8 * 2;  // 2048

template <int EC>
struct DwgBulk {
  static constexpr int G = EC == 8 ? 4 : 2;
  static constexpr int kThreads = G * kFastDwgThreads;
};

size_t dwg_bulk_smem(int tps, int ec) {
  return static_cast<size_t>(kDwgBulkStages) * kDwgBulkRows * kDwgBulkRowBytes + 128 +
         static_cast<size_t>(tps) * ec * sizeof(float);
}

template <int EC>
__global__ void __launch_bounds__(DwgBulk<EC>::kThreads, 1)
bwd_dwg_bulk(const __nv_bfloat16* __restrict__ x, const float* __restrict__ dl, int Tn, int d, int E,
             int tok_per_split, float* __restrict__ part, Control* ctl) {
  pdl_begin();
  constexpr int G = DwgBulk<EC>::G, NT = DwgBulk<EC>::kThreads;
  static_assert(static_cast<size_t>(G - 1) * kFastDwgThreads * 8 * EC * 4 <=
                    static_cast<size_t>(kDwgBulkStages) * kDwgBulkRows * kDwgBulkRowBytes,
                "the groups' sums fit in the ring");
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ __align__(8) uint64_t full[kDwgBulkStages], empty[kDwgBulkStages];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm) + 127) & ~uintptr_t(127));
  float* dls = reinterpret_cast<float*>(ring + kDwgBulkStages * kDwgBulkRows * kDwgBulkRowBytes);
  const int tid = threadIdx.x;
  const int grp = tid / kFastDwgThreads, gt = tid - grp * kFastDwgThreads;
  const int c0 = blockIdx.x * kFastDwgThreads * 8;
  const int ncol = min(kFastDwgThreads * 8, d - c0);
  const uint32_t rowb = static_cast<uint32_t>(ncol) * 2;  // a multiple of 16 (d % 8 == 0)
  const int tb = blockIdx.y * tok_per_split;
  const int n = max(0, min(Tn, tb + tok_per_split) - tb);
  const int nstg = (n + kDwgBulkRows - 1) / kDwgBulkRows;
  if (tid == 0) {
    for (int i = 0; i < kDwgBulkStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], NT);
    }
    fence_mbar_init();
  }
  for (int i = tid; i < n * EC; i += NT) {
    const int tt = i / EC, e = i - tt * EC;
    dls[i] = e < E ? __ldg(dl + static_cast<size_t>(tb + tt) * E + e) : 0.f;
  }
  __syncthreads();
  auto issue = [&](int st) {
    const int slot = st % kDwgBulkStages, r0 = st * kDwgBulkRows;
    const int nr = min(kDwgBulkRows, n - r0);
    mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(nr) * rowb);
    for (int r = 0; r < nr; ++r)
      bulk_load(ring + (slot * kDwgBulkRows + r) * kDwgBulkRowBytes,
                x + static_cast<size_t>(tb + r0 + r) * d + c0, rowb, &full[slot]);
  };
  if (tid == 0)
    for (int st = 0; st < nstg && st < kDwgBulkStages; ++st) issue(st);
  float acc[8][EC];
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int e = 0; e < EC; ++e) acc[j][e] = 0.f;
  const bool mine = gt * 8 < ncol;
  int issued = min(nstg, kDwgBulkStages);
  bool ok = true;
  for (int st = 0; st < nstg; ++st) {
    const int slot = st % kDwgBulkStages;
    if (!mbar_wait_bounded(&full[slot], static_cast<uint32_t>(st / kDwgBulkStages) & 1u)) {
      set_error(ctl, MOE_DEVERR_TIMEOUT);
      ok = false;
      break;
    }
    const int nr = min(kDwgBulkRows, n - st * kDwgBulkRows);
    if (mine) {
      const uint8_t* rows = ring + slot * kDwgBulkRows * kDwgBulkRowBytes + gt * 16;
#pragma unroll 2
      for (int r = grp; r < nr; r += G) {
        float xv[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(rows + r * kDwgBulkRowBytes), xv);
        const float* g = dls + (st * kDwgBulkRows + r) * EC;
#pragma unroll
        for (int e = 0; e < EC; ++e) {
          const float ge = g[e];
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[j][e] = fmaf(xv[j], ge, acc[j][e]);
        }
      }
    }
    mbar_arrive(&empty[slot]);
    if (tid == 0 && issued < nstg) {
      // the slot is free once every thread has read this stage
      if (!mbar_wait_bounded(&empty[slot], static_cast<uint32_t>(st / kDwgBulkStages) & 1u)) {
        set_error(ctl, MOE_DEVERR_TIMEOUT);
        ok = false;
        break;
      }
      issue(issued);
      ++issued;
    }
  }
  if (tid == 0) {
    // every copy issued must have landed before the ring is reused or the
    // block leaves: wait for the last stage issued into each slot
    for (int slot = 0; slot < kDwgBulkStages && slot < issued; ++slot) {
      const int last = slot + ((issued - 1 - slot) / kDwgBulkStages) * kDwgBulkStages;
      if (!mbar_wait_bounded(&full[slot], static_cast<uint32_t>(last / kDwgBulkStages) & 1u))
        set_error(ctl, MOE_DEVERR_TIMEOUT);
    }
  }
  __syncthreads();  // every thread is done with the ring: it holds the groups' sums now
  float* red = reinterpret_cast<float*>(ring);  // [G - 1][128 threads][8][EC]
  if (grp > 0 && mine) {
    float* dst = red + (static_cast<size_t>(grp - 1) * kFastDwgThreads + gt) * 8 * EC;
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < EC; e += 4)
        *reinterpret_cast<float4*>(dst + j * EC + e) =
            make_float4(acc[j][e], acc[j][e + 1], acc[j][e + 2], acc[j][e + 3]);
  }
  __syncthreads();
  if (grp != 0 || !mine || !ok) return;
#pragma unroll
  for (int q = 1; q < G; ++q) {
    const float* src = red + (static_cast<size_t>(q - 1) * kFastDwgThreads + gt) * 8 * EC;
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < EC; ++e) acc[j][e] += src[j * EC + e];
  }
  // the 8 columns' E values are 8 * E consecutive floats of the partial
  float* dst = part + (static_cast<size_t>(blockIdx.y) * d + c0 + gt * 8) * E;
  if (E == EC) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < EC; e += 4)
        *reinterpret_cast<float4*>(dst + j * EC + e) =
            make_float4(acc[j][e], acc[j][e + 1], acc[j][e + 2], acc[j][e + 3]);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < EC; ++e)
        if (e < E) dst[j * E + e] = acc[j][e];
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
  // bf16 with at most 16 experts: the streaming kernels (16-byte row access;
  // dWg through the bulk-copy ring while a split's d_logits fit beside it)
  const bool fast = dt == MOE_BF16 && E <= 16 && d % 8 == 0;
  const int fxb = (d + kFastDwgThreads * 8 - 1) / (kFastDwgThreads * 8);
  const int fns = std::max(1, std::min(dwg_splits(T, d, E), num_sms() / fxb));
  const int ftps = T > 0 ? (T + fns - 1) / fns : 0;
  const bool fast_dwg = fast && dwg_bulk_smem(std::max(ftps, 1), E <= 8 ? 8 : 16) <= 200 * 1024;
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
    if (dx != nullptr && fast) {
      const dim3 g((d + kFastThreads * 8 - 1) / (kFastThreads * 8), (T + kFastTok - 1) / kFastTok);
      auto kern = E <= 8 ? bwd_dx_fast<8> : bwd_dx_fast<16>;
      const size_t dsm = dx_fast_smem(E <= 8 ? 8 : 16);
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(dsm));
      err = launch_pdl(kern, g, dim3(kFastThreads), dsm, s, false, static_cast<const float*>(dl),
                       static_cast<const __nv_bfloat16*>(wg), T, d, E, static_cast<__nv_bfloat16*>(dx));
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
  if (d_wg != nullptr && fast_dwg) {
    // one block per SM: the column slices times the token splits
    const int xb = fxb, ns = fns, tps = ftps;
    const int ec = E <= 8 ? 8 : 16;
    const size_t smem = dwg_bulk_smem(std::max(tps, 1), ec);
    auto kern = ec == 8 ? bwd_dwg_bulk<8> : bwd_dwg_bulk<16>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    const int nthr = ec == 8 ? DwgBulk<8>::kThreads : DwgBulk<16>::kThreads;
    err = launch_pdl(kern, dim3(xb, ns), dim3(nthr), smem, s, false,
                     static_cast<const __nv_bfloat16*>(x), static_cast<const float*>(dl), T, d, E, tps,
                     part, ctl);
    if (err != cudaSuccess) return err;
    const long long n = static_cast<long long>(d) * E;
    const int rg = static_cast<int>(std::min<long long>((n + 255) / 256, 8LL * num_sms()));
    err = launch_pdl(bwd_dwg_reduce, dim3(std::max(rg, 1)), dim3(256), 0, s, false,
                     static_cast<const float*>(part), ns, n, d_wg);
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
