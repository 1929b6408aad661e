// Router: gate GEMM (fp32 accumulate), softmax over E, top-k by selection
// (ties to the lower expert index), renormalisation of the k weights, and the
// load-balance loss aux = E * sum_i f_i * P_i.
//
// Sources: "ops-transformer MoE operators" blog, 实现 (MoEGatingForward:
// Softmax, TopK by a selection rather than a sort, NormalizeWeights);
// "MoE Router" page (Linear(hidden, E, bias=False) -> softmax -> topk ->
// renormalise); "MegaBlocks 01", section 1 (bias-free linear router).
//
// Paths:
//  * bf16 with E a multiple of 8 (E <= 32) or of 64: the gate GEMM runs on the
//    tcgen05 tensor cores (router_tc: x streamed once by TMA, fp32 split-K
//    partial logits to an L2-resident scratch), then router_select (a warp per
//    token) adds the partials in order and routes.
//  * fp32 with E <= 8: one fused CUDA-core kernel (router_fused_e8).
//  * otherwise: a tiled CUDA-core GEMM for the logits, then router_select.
// Every path leaves per-block aux partials (expert-major); aux_reduce sums them
// in a fixed order (one block per expert, then the last block over experts),
// so the loss is deterministic.
#include "common.cuh"
#include "ptx.cuh"
#include <cfloat>
#include <cmath>
#include <algorithm>

namespace moe {

namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ bool better(float va, int ea, float vb, int eb) {
  return va > vb || (va == vb && ea < eb);
}

// This block's aux partials (per-expert probability sums and slot counts),
// expert-major: part[e * ldb + block]. ldb = the largest grid of any router
// kernel (route_max_blocks), so every path shares one layout.
__device__ __forceinline__ void block_write_partials(const float* blk_p, const int32_t* blk_c,
                                                     float* part_p, int32_t* part_c, int ldb,
                                                     int E) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    part_p[static_cast<size_t>(e) * ldb + blockIdx.x] = blk_p[e];
    part_c[static_cast<size_t>(e) * ldb + blockIdx.x] = blk_c[e];
  }
}

// aux = E * sum_e f_e * P_e with f_e = count_e / (T*k), P_e = (sum_t p_te) / T.
// Block e sums expert e's nblk partials (thread i: blocks i, i+256, ... in
// order, float64; then a fixed tree) and writes its term; the last block to
// finish (ticket) adds the E terms with a fixed tree. Deterministic.
constexpr int kAuxThreads = 256;

__global__ void __launch_bounds__(kAuxThreads)
aux_reduce(const float* __restrict__ part_p, const int32_t* __restrict__ part_c,
           const float* __restrict__ part_z, int ldb, int nblk, int E, int T, int k,
           double* __restrict__ terms, float* __restrict__ aux, float* __restrict__ z_out,
           Control* ctl) {
  pdl_begin();
  __shared__ double sp[kAuxThreads];
  __shared__ long long sc[kAuxThreads];
  __shared__ bool is_last;
  const int e = blockIdx.x;
  double ps = 0.0;
  long long cs = 0;
  for (int b = threadIdx.x; b < nblk; b += kAuxThreads) {
    ps += static_cast<double>(part_p[static_cast<size_t>(e) * ldb + b]);
    cs += part_c[static_cast<size_t>(e) * ldb + b];
  }
  sp[threadIdx.x] = ps;
  sc[threadIdx.x] = cs;
  __syncthreads();
  for (int s = kAuxThreads / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) { sp[threadIdx.x] += sp[threadIdx.x + s]; sc[threadIdx.x] += sc[threadIdx.x + s]; }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    terms[e] = T > 0 ? (static_cast<double>(sc[0]) / (static_cast<double>(T) * k)) * (sp[0] / T) : 0.0;
    __threadfence();
    is_last = atomicAdd(&ctl->route_ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  sp[threadIdx.x] = threadIdx.x < E ? __ldcg(terms + threadIdx.x) : 0.0;
  __syncthreads();
  for (int s = kAuxThreads / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) sp[threadIdx.x] += sp[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) *aux = static_cast<float>(E * sp[0]);
  if (z_out != nullptr) {  // z-loss: the blocks' partials in a fixed order, then / T
    __syncthreads();
    double zs = 0.0;
    for (int b = threadIdx.x; b < nblk; b += kAuxThreads) zs += static_cast<double>(__ldcg(part_z + b));
    sp[threadIdx.x] = zs;
    __syncthreads();
    for (int s = kAuxThreads / 2; s > 0; s >>= 1) {
      if (threadIdx.x < s) sp[threadIdx.x] += sp[threadIdx.x + s];
      __syncthreads();
    }
    if (threadIdx.x == 0) *z_out = T > 0 ? static_cast<float>(sp[0] / T) : 0.f;
  }
  if (threadIdx.x == 0) ctl->route_ticket = 0u;
}

// ---------------------------------------------------------------- fused, E <= 8
template <typename Tin>
struct VecTraits;
template <> struct VecTraits<float> {
  static constexpr int kVec = 4;
  static __device__ __forceinline__ void unpack(const uint4& u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
};


// Fused router for E <= 8.
//
// Block = 12 warps = 6 slices of d x 2 token quads: warp (slice, quad) takes 4
// tokens and one sixth of d, so a block works on 8 tokens and each SM keeps
// 12 warps' x loads in flight. Wg is staged once per block in shared memory as
// fp32 pairs: for row pair p = (2p, 2p+1) and expert e the float2
// (Wg[2p][e], Wg[2p+1][e]); a lane's 16-byte x slice (8 bf16 = 4 row pairs)
// then meets 4 pair-rows of 64 bytes, read with an XOR swizzle so that the 8
// lanes of a quarter-warp hit 8 different bank groups. Products use the packed
// fma.rn.f32x2 (even rows in .x, odd rows in .y; the two halves are added at
// the end). Each warp's partial logits are reduce-scattered (lane l: token l/8,
// expert l%8), the slices are added in slice order through shared memory,
// and the quads' 8-lane groups do softmax / top-k / renormalisation.
constexpr int kFusedSlices = 6;
constexpr int kFusedQuads = 2;
constexpr int kFusedTokensPerGroup = 4 * kFusedQuads;
constexpr int kFusedThreads = 32 * kFusedSlices * kFusedQuads;

__device__ __forceinline__ void fma2(float2& acc, float2 a, float2 b) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(r)
      : "l"(*reinterpret_cast<const unsigned long long*>(&a)),
        "l"(*reinterpret_cast<const unsigned long long*>(&b)),
        "l"(*reinterpret_cast<const unsigned long long*>(&acc)));
  acc = *reinterpret_cast<const float2*>(&r);
}

// Byte offset of 16-byte chunk c (0..15) of the 256-byte block of 4 pair-rows
// owned by slice position g (pair-rows 4g .. 4g+3).
__device__ __forceinline__ uint32_t wg_chunk_off(uint32_t g, uint32_t c) {
  return g * 256u + 16u * (c ^ (g & 7u));
}

template <typename Tin>
__global__ void __launch_bounds__(kFusedThreads, 1)
router_fused_e8(const Tin* __restrict__ x, const Tin* __restrict__ wg, const float* __restrict__ bias,
                int T, int d, int E, int k, int32_t* __restrict__ idx_out, float* __restrict__ w_out,
                float* __restrict__ logits_out, float* __restrict__ probs_out,
                float* __restrict__ part_p, int32_t* __restrict__ part_c, int ldb,
                Control* ctl) {
  pdl_begin();
  constexpr int V = VecTraits<Tin>::kVec;  // elements per 16-byte x load: 8 (bf16) or 4 (fp32)
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ float slice_part[kFusedSlices][kFusedQuads][32];
  __shared__ float blk_p[kFusedQuads][8];
  __shared__ int32_t blk_c[kFusedQuads][8];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int slice = warp / kFusedQuads, quad = warp % kFusedQuads;

  // ---- stage Wg: row pairs (zero for experts >= E and for a missing odd row)
  const int npairs = (d + 1) / 2;
  if (sizeof(Tin) == 2 && E == 8) {
    // two 16-byte rows per pair-row, all loads of a thread in flight together
    const uint4* src = reinterpret_cast<const uint4*>(wg);
#pragma unroll 4
    for (int p = threadIdx.x; p < npairs; p += kFusedThreads) {
      const uint4 r0 = __ldg(src + 2 * p), r1 = __ldg(src + 2 * p + 1);
      const uint32_t a[4] = {r0.x, r0.y, r0.z, r0.w}, b[4] = {r1.x, r1.y, r1.z, r1.w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // experts 2c, 2c+1
        const float4 v = make_float4(__uint_as_float(a[c] << 16), __uint_as_float(b[c] << 16),
                                     __uint_as_float(a[c] & 0xffff0000u),
                                     __uint_as_float(b[c] & 0xffff0000u));
        *reinterpret_cast<float4*>(smem_raw + wg_chunk_off(p >> 2, ((p & 3) << 2) | c)) = v;
      }
    }
  } else
  for (int i = threadIdx.x; i < npairs * 8; i += kFusedThreads) {
    const int p = i >> 3, e = i & 7;
    float w0 = 0.f, w1 = 0.f;
    if (e < E) {
      w0 = Elem<Tin>::to_f32(wg[static_cast<size_t>(2 * p) * E + e]);
      if (2 * p + 1 < d) w1 = Elem<Tin>::to_f32(wg[static_cast<size_t>(2 * p + 1) * E + e]);
    }
    // pair-row p, expert e: chunk (p % 4) * 4 + e / 2 of group p / 4, half e % 2
    const uint32_t off = wg_chunk_off(p >> 2, ((p & 3) << 2) | (e >> 1)) + (e & 1) * 8;
    *reinterpret_cast<float2*>(smem_raw + off) = make_float2(w0, w1);
  }
  __syncthreads();

  const int tq = lane >> 3;  // token of the quad after the reduce-scatter
  const int e = lane & 7;
  const bool e_ok = e < E;
  const float b_e = (bias != nullptr && e_ok) ? bias[e] : 0.f;
  float psum = 0.f;
  int cnt = 0;
  // this slice's share of d, cut at multiples of 8 elements (one 16-byte group of 4 pairs)
  const int nvec8 = d / 8;  // whole 8-element vectors (d % 8 == 0 here, see use_fused)
  const int per = (nvec8 + kFusedSlices - 1) / kFusedSlices;
  const int v_lo = min(nvec8, slice * per), v_hi = min(nvec8, v_lo + per);

  const int groups = (T + kFusedTokensPerGroup - 1) / kFusedTokensPerGroup;
  for (int g = blockIdx.x; g < groups; g += gridDim.x) {
    const int t_base = g * kFusedTokensPerGroup + quad * 4;
    float2 acc[4][8];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[q][j] = make_float2(0.f, 0.f);

    constexpr int kUnroll = 2;
    for (int vb = v_lo + lane; vb < v_hi; vb += 32 * kUnroll) {
      uint4 raw[kUnroll][4][8 / V];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int v = vb + 32 * u;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int t = t_base + q;
#pragma unroll
          for (int h = 0; h < 8 / V; ++h) {
            raw[u][q][h] = make_uint4(0, 0, 0, 0);
            if (t < T && v < v_hi)
              raw[u][q][h] = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d +
                                                                   static_cast<size_t>(v) * 8 + h * V));
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int v = vb + 32 * u;
        if (v >= v_hi) break;
        const uint32_t grp = static_cast<uint32_t>(v);  // pair-rows 4v .. 4v+3
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
          // row pair pp of the 4 tokens' 8-element slices
          float2 xq[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if constexpr (sizeof(Tin) == 2) {
              const uint32_t wv = pp == 0 ? raw[u][q][0].x : pp == 1 ? raw[u][q][0].y
                                : pp == 2 ? raw[u][q][0].z : raw[u][q][0].w;
              xq[q] = make_float2(__uint_as_float(wv << 16), __uint_as_float(wv & 0xffff0000u));
            } else {
              const uint4& r4 = raw[u][q][pp >> 1];
              xq[q] = (pp & 1) ? make_float2(__uint_as_float(r4.z), __uint_as_float(r4.w))
                               : make_float2(__uint_as_float(r4.x), __uint_as_float(r4.y));
            }
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) {  // experts 2c, 2c+1
            const float4 w = *reinterpret_cast<const float4*>(smem_raw + wg_chunk_off(grp, (pp << 2) | c));
            const float2 wa = make_float2(w.x, w.y), wb = make_float2(w.z, w.w);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              fma2(acc[q][2 * c], xq[q], wa);
              fma2(acc[q][2 * c + 1], xq[q], wb);
            }
          }
        }
      }
    }
    // even + odd halves, then reduce-scatter: lane l holds the sum of value l
    float a[32];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int j = 0; j < 8; ++j) a[q * 8 + j] = acc[q][j].x + acc[q][j].y;
#pragma unroll
    for (int half = 16; half >= 1; half >>= 1) {
      const bool upper = (lane & half) != 0;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float send = upper ? a[i] : a[i + half];
        const float keep = upper ? a[i + half] : a[i];
        a[i] = keep + __shfl_xor_sync(kFull, send, half);
      }
    }
    slice_part[slice][quad][lane] = a[0];
    __syncthreads();
    if (slice == 0) {
      const int t = t_base + tq;
      const bool t_ok = t < T;
      float lg = 0.f;
#pragma unroll
      for (int sl = 0; sl < kFusedSlices; ++sl) lg += slice_part[sl][quad][lane];
      float v = e_ok ? lg + b_e : -INFINITY;
      if (logits_out != nullptr && t_ok && e_ok) logits_out[static_cast<size_t>(t) * E + e] = v;

      // softmax inside the 8-lane group of token t
      float m = v;
#pragma unroll
      for (int off = 4; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
      const float ex = e_ok ? expf(v - m) : 0.f;
      float sm = ex;
#pragma unroll
      for (int off = 4; off >= 1; off >>= 1) sm += __shfl_xor_sync(kFull, sm, off);
      const float p = ex / sm;
      if (probs_out != nullptr && t_ok && e_ok) probs_out[static_cast<size_t>(t) * E + e] = p;
      if (t_ok && e_ok) psum += p;

      // top-k by k rounds of a group arg-max
      bool taken = !e_ok;
      float wsum = 0.f;
      int my_e = 0;
      float my_p = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < k) {
          float bv = taken ? -INFINITY : v;
          int be = taken ? 0x7fffffff : e;
#pragma unroll
          for (int off = 4; off >= 1; off >>= 1) {
            const float ov = __shfl_xor_sync(kFull, bv, off);
            const int oe = __shfl_xor_sync(kFull, be, off);
            if (better(ov, oe, bv, be)) { bv = ov; be = oe; }
          }
          if (be >= E || be < 0) {
            if (t_ok && e == 0) set_error(ctl, MOE_DEVERR_EXPERT_RANGE);
            be = 0;
          }
          const float pb = __shfl_sync(kFull, p, (lane & ~7) | be);
          if (e == be) {
            taken = true;
            if (t_ok) ++cnt;
          }
          wsum += pb;
          if (e == j) { my_e = be; my_p = pb; }
        }
      }
      if (t_ok && e < k) {
        idx_out[static_cast<size_t>(t) * k + e] = my_e;
        w_out[static_cast<size_t>(t) * k + e] = my_p / wsum;
      }
    }
    __syncthreads();  // slice_part is rewritten by the next group
  }
  // Warp totals per expert: lanes e, e+8, e+16, e+24 hold the same expert.
  if (slice == 0) {
    psum += __shfl_xor_sync(kFull, psum, 8);
    psum += __shfl_xor_sync(kFull, psum, 16);
    cnt += __shfl_xor_sync(kFull, cnt, 8);
    cnt += __shfl_xor_sync(kFull, cnt, 16);
    if (lane < 8) {
      blk_p[quad][lane] = psum;
      blk_c[quad][lane] = cnt;
    }
  }
  __syncthreads();
  __shared__ float tot_p[8];
  __shared__ int32_t tot_c[8];
  if (threadIdx.x < 8) {
    float s = 0.f;
    int c = 0;
    for (int w = 0; w < kFusedQuads; ++w) { s += blk_p[w][threadIdx.x]; c += blk_c[w][threadIdx.x]; }
    tot_p[threadIdx.x] = s;
    tot_c[threadIdx.x] = c;
  }
  __syncthreads();
  block_write_partials(tot_p, tot_c, part_p, part_c, ldb, E);
}

// ---------------------------------------------------------------- general path
// logits[T, E] = x[T, d] * Wg[d, E], 64x64 tiles, 256 threads with 4x4 each.
template <typename Tin>
__global__ void __launch_bounds__(256)
router_gemm_tiled(const Tin* __restrict__ x, const Tin* __restrict__ wg, int T, int d, int E,
                  float* __restrict__ out) {
  pdl_begin();
  __shared__ float xs[32][64 + 4];
  __shared__ float ws[32][64 + 4];
  const int t0 = blockIdx.x * 64, e0 = blockIdx.y * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < d; k0 += 32) {
    for (int i = threadIdx.x; i < 64 * 32; i += 256) {
      const int tok = i >> 5, kk = i & 31;
      const int t = t0 + tok, kg = k0 + kk;
      xs[kk][tok] = (t < T && kg < d) ? Elem<Tin>::to_f32(x[static_cast<size_t>(t) * d + kg]) : 0.f;
    }
    for (int i = threadIdx.x; i < 64 * 32; i += 256) {
      const int kk = i >> 6, ee = i & 63;
      const int kg = k0 + kk, eg = e0 + ee;
      ws[kk][ee] = (eg < E && kg < d) ? Elem<Tin>::to_f32(wg[static_cast<size_t>(kg) * E + eg]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = xs[kk][ty * 4 + i]; b[i] = ws[kk][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int eg = e0 + tx * 4 + j;
      if (eg < E) out[static_cast<size_t>(t) * E + eg] = acc[i][j];
    }
  }
}

// An unsigned key with the order of the float v: sign-magnitude to offset
// binary. -0 is taken as +0 first, so keys are equal exactly when the floats
// compare equal; NaN gets key 0, below every number (never selected, as a
// comparison would not select it).
__device__ __forceinline__ uint32_t order_key(float v) {
  if (v != v) return 0u;
  const uint32_t u = v == 0.0f ? 0u : __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// One token's routing by one warp: lane l holds the logits (bias included) of
// experts l + 32q, q < EPL (-inf for e >= E). Softmax over E, top-k by k
// rounds of a warp arg-max (ties to the lower expert), renormalised weights;
// accumulates the token's probabilities and choices into the lane's aux sums.
// A round's arg-max is two warp reductions: the largest key of the lanes'
// best untaken logits, then the lowest expert among the lanes that hold it.
template <int EPL>
__device__ __forceinline__ float warp_route_token(const float (&v)[EPL], int E, int k, int lane,
                                                 size_t t, int32_t* __restrict__ idx_out,
                                                 float* __restrict__ w_out,
                                                 float* __restrict__ logits_out,
                                                 float* __restrict__ probs_out,
                                                 float (&psum)[EPL], int (&cnt)[EPL],
                                                 float inv_tau, Control* ctl) {
#pragma unroll
  for (int q = 0; q < EPL; ++q) {
    const int e = lane + 32 * q;
    if (logits_out != nullptr && e < E) logits_out[t * E + e] = v[q];
  }
  uint32_t mk = 0;
#pragma unroll
  for (int q = 0; q < EPL; ++q) mk = max(mk, order_key(v[q]));
  const float m = key_value(__reduce_max_sync(kFull, mk));
  float ex[EPL], s = 0.f;
#pragma unroll
  for (int q = 0; q < EPL; ++q) {
    ex[q] = (lane + 32 * q < E) ? expf((v[q] - m) * inv_tau) : 0.f;
    s += ex[q];
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(kFull, s, off);
  float p[EPL];
#pragma unroll
  for (int q = 0; q < EPL; ++q) {
    const int e = lane + 32 * q;
    p[q] = ex[q] / s;
    if (e < E) {
      psum[q] += p[q];
      if (probs_out != nullptr) probs_out[t * E + e] = p[q];
    }
  }
  unsigned taken = 0;
  float wsum = 0.f;
  int my_e = 0;
  float my_p = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < k) {
      // the lane's best untaken expert (q ascending, strict >: ties keep the
      // lower expert); key 0 is below every logit's key and means none
      uint32_t bk = 0;
      int be = 0x7fffffff;
#pragma unroll
      for (int q = 0; q < EPL; ++q) {
        const int e = lane + 32 * q;
        const uint32_t key = order_key(v[q]);
        if (e < E && !((taken >> q) & 1u) && key > bk) { bk = key; be = e; }
      }
      const uint32_t wk = __reduce_max_sync(kFull, bk);
      be = static_cast<int>(__reduce_min_sync(kFull, bk == wk ? static_cast<uint32_t>(be) : 0xffffffffu));
      if (be >= E || be < 0) {
        if (lane == 0) set_error(ctl, MOE_DEVERR_EXPERT_RANGE);
        be = 0;
      }
      const int owner = be & 31, qq = be >> 5;
      float pv = 0.f;
#pragma unroll
      for (int q = 0; q < EPL; ++q)
        if (q == qq) pv = p[q];
      pv = __shfl_sync(kFull, pv, owner);
      if (lane == owner) {
#pragma unroll
        for (int q = 0; q < EPL; ++q)
          if (q == qq) { taken |= 1u << q; ++cnt[q]; }
      }
      wsum += pv;
      if (lane == j) { my_e = be; my_p = pv; }
    }
  }
  if (lane < k) {
    idx_out[t * k + lane] = my_e;
    w_out[t * k + lane] = my_p / wsum;
  }
  // log-sum-exp of the logits the softmax sees (l / tau; the z-loss term),
  // the same in every lane
  return m * inv_tau + logf(s);
}

// Warp per token: lane l holds experts l + 32q, q < EPL. The logits are the
// sum of KS partial [T, E] buffers (stride T*E), added in order, plus the bias.
constexpr int kSelectWarps = 8;
constexpr int kSelectTokensPerWarp = 2;
constexpr int kSelectTokensPerBlock = kSelectWarps * kSelectTokensPerWarp;

template <int EPL>
__global__ void __launch_bounds__(kSelectWarps * 32)
router_select(const float* __restrict__ logits_in, int KS, const float* __restrict__ bias,
              const float* __restrict__ noise, int T, int E, int k, int32_t* __restrict__ idx_out,
              float* __restrict__ w_out, float* __restrict__ logits_out,
              float* __restrict__ probs_out, float* __restrict__ part_p,
              int32_t* __restrict__ part_c, float* __restrict__ part_z, int ldb, float inv_tau,
              Control* ctl) {
  pdl_begin();
  __shared__ float zw[kSelectWarps];
  __shared__ float blk_p_w[kSelectWarps][256];
  __shared__ int32_t blk_c_w[kSelectWarps][256];
  __shared__ float tot_p[256];
  __shared__ int32_t tot_c[256];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float psum[EPL];
  int cnt[EPL];
  float bq[EPL];
#pragma unroll
  for (int q = 0; q < EPL; ++q) {
    psum[q] = 0.f;
    cnt[q] = 0;
    const int e = lane + 32 * q;
    bq[q] = (bias != nullptr && e < E) ? bias[e] : 0.f;
  }
  const size_t plane = static_cast<size_t>(T) * E;
  float zacc = 0.f;  // this warp's sum of squared log-sum-exp (z-loss)
  const int t_begin = blockIdx.x * kSelectTokensPerBlock;
  const int t_end = min(T, t_begin + kSelectTokensPerBlock);
  for (int t = t_begin + warp; t < t_end; t += kSelectWarps) {
    float pv[8][EPL];
#pragma unroll
    for (int src = 0; src < 8; ++src)
#pragma unroll
      for (int q = 0; q < EPL; ++q) {
        const int e = lane + 32 * q;
        pv[src][q] = (src < KS && e < E)
                         ? __ldcg(logits_in + src * plane + static_cast<size_t>(t) * E + e) : 0.f;
      }
    float v[EPL];
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
      float acc = 0.f;
#pragma unroll
      for (int src = 0; src < 8; ++src)
        if (src < KS) acc += pv[src][q];
      const int e = lane + 32 * q;
      v[q] = e < E ? acc + bq[q] : -INFINITY;
      if (noise != nullptr && e < E) v[q] += __ldg(noise + static_cast<size_t>(t) * E + e);
    }
    const float lse = warp_route_token<EPL>(v, E, k, lane, static_cast<size_t>(t), idx_out, w_out,
                                            logits_out, probs_out, psum, cnt, inv_tau, ctl);
    zacc += lse * lse;
  }
  if (lane == 0) zw[warp] = zacc;
#pragma unroll
  for (int q = 0; q < EPL; ++q) {
    const int e = lane + 32 * q;
    if (e < E) { blk_p_w[warp][e] = psum[q]; blk_c_w[warp][e] = cnt[q]; }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float a = 0.f;
    int c = 0;
    for (int w = 0; w < kSelectWarps; ++w) { a += blk_p_w[w][e]; c += blk_c_w[w][e]; }
    tot_p[e] = a;
    tot_c[e] = c;
  }
  __syncthreads();
  block_write_partials(tot_p, tot_c, part_p, part_c, ldb, E);
  if (part_z != nullptr && threadIdx.x == 0) {
    float z = 0.f;
    for (int w = 0; w < kSelectWarps; ++w) z += zw[w];
    part_z[blockIdx.x] = z;
  }
}

// ---------------------------------------------------------------- tensor cores
// The gate GEMM on tcgen05 for bf16 layers. CTA (tile, ks) takes 128 tokens
// and the d-range [ks*dk, (ks+1)*dk). Warp 0 streams the x tile (TMA, 128x64,
// 128-byte swizzle) through a 4-stage ring; warp 1 issues M=128, N=Epad (E
// rounded up to 16), K=16 MMAs into tensor memory. Wg is either TMA-streamed
// beside x as the MN-major operand (E a multiple of 64, the expert GEMM's B
// path) or, for E <= 32, transposed once into shared memory as a K-major
// operand (the first ring stages are already loading meanwhile). The four
// warps then copy their 32 accumulator rows to the fp32 partial buffer
// logits[ks][t][e]; router_select adds the KS partials in ks order. The ring
// has as many stages (up to kTcStages) as shared memory holds.
constexpr int kTcStages = 8;
constexpr int kTcThreads = 128;
constexpr int kMaxKS = 8;  // largest split of d over the CTAs of one token tile

struct RouterTcArgs {
  int T, d, E, Epad, KS, dk, stages;
  int tmem_cap;             // tensor-memory columns one CTA may take (512 / CTAs per SM)
  int sub;                  // persistent kernel: k-blocks per ring stage, loaded together
  const __nv_bfloat16* wg;  // [d, E] (staged path)
  float* partial;           // [KS][T][E] (unfused)
  Control* ctl;
  // fused selection (kFuseE != 0): the router's outputs and aux partials
  const float* bias;
  int k, ntile, ldb;
  int32_t* idx;
  float *w, *logits, *probs, *part_p, *aux;
  int32_t* part_c;
  const float* noise;  // [T, E] added to the logits, or null
  float* part_z;       // per-tile z-loss partials, or null (no z-loss)
  float* z_out;        // the z-loss, or null
  float inv_tau;       // 1 / the softmax temperature (1: the plain router)
};

// Fused selection, E <= 32. The KS CTAs of one 128-token tile run as a
// cluster: CTA ks > 0 leaves its partial logits in its own shared memory and
// the leader (ks = 0) adds them in ks order through distributed shared memory,
// then the bias (the order router_select uses, so the logits are the same).
// Leader thread r owns token tile*128 + r: softmax, k rounds of arg-max (ties
// to the lower expert), renormalisation. The tile's aux partials
// (probability sums and selection counts per expert) go to part[e][tile];
// the last tile to finish (ticket) adds them in tile order and writes the
// loss. EW (8, 16 or 32) is E rounded up: the per-token loops are that wide.
constexpr int kFuseMaxE = 32;

template <int EW>
struct FuseCfg {
  static constexpr int kStride = EW + 4;            // floats per shared row (16-byte aligned)
  static constexpr int kParts = kTcThreads / EW;    // threads per expert in the reductions
  static constexpr size_t kScratch = 2 * 128 * kStride * 4 + 128 * 4 + kTcThreads * 8;
};

// Thread r: the sum over accumulator slots (in slot order) of the first EW
// columns of its row (trow = the row's tensor-memory address).
template <int EW>
__device__ __forceinline__ void slot_sums(uint32_t trow, int nslot, int Epad, float (&v)[EW]) {
#pragma unroll
  for (int h = 0; h < (EW + 15) / 16; ++h) {
    float sum[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) sum[i] = 0.f;
    for (int sl = 0; sl < nslot; ++sl) {
      uint32_t u[16];
      tmem_ld_32x32b_x16(trow + sl * Epad + h * 16, u);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) sum[i] += __uint_as_float(u[i]);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (h * 16 + i < EW) v[h * 16 + i] = sum[i];
  }
}

// The split over d (KS > 1): CTA ks > 0 leaves its row sums in its own shared
// memory (red) and the leader (ks = 0) adds them in ks order through
// distributed shared memory. Every thread of every CTA of the cluster reaches
// both cluster barriers.
template <int EW>
__device__ __forceinline__ void cluster_row_sums(int KS, int ks, int r, float* red, float (&v)[EW]) {
  using F = FuseCfg<EW>;
  if (ks != 0) {
#pragma unroll
    for (int e = 0; e < EW; e += 4)
      *reinterpret_cast<float4*>(red + r * F::kStride + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
  }
  cluster_sync();
  if (ks == 0) {
    const uint32_t own = smem_u32(red + r * F::kStride);
    if constexpr (EW == 8) {
      // all peers' rows requested at once (one round trip), added in ks order
      float4 q[kMaxKS - 1][2];
#pragma unroll
      for (int src = 1; src < kMaxKS; ++src)
        if (src < KS) {
          const uint32_t base = mapa_shared(own, static_cast<uint32_t>(src));
          q[src - 1][0] = ld_shared_cluster_f32x4(base);
          q[src - 1][1] = ld_shared_cluster_f32x4(base + 16u);
        }
#pragma unroll
      for (int src = 1; src < kMaxKS; ++src)
        if (src < KS) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            v[4 * h] += q[src - 1][h].x;
            v[4 * h + 1] += q[src - 1][h].y;
            v[4 * h + 2] += q[src - 1][h].z;
            v[4 * h + 3] += q[src - 1][h].w;
          }
        }
    } else {
      for (int src = 1; src < KS; ++src) {
        const uint32_t base = mapa_shared(own, static_cast<uint32_t>(src));
        float4 q[EW / 4];
#pragma unroll
        for (int e = 0; e < EW / 4; ++e) q[e] = ld_shared_cluster_f32x4(base + 16u * e);
#pragma unroll
        for (int e = 0; e < EW / 4; ++e) {
          v[4 * e] += q[e].x;
          v[4 * e + 1] += q[e].y;
          v[4 * e + 2] += q[e].z;
          v[4 * e + 3] += q[e].w;
        }
      }
    }
  }
  cluster_sync();  // the other CTAs keep their buffers until the leader has read them
}

// Selection and aux partials of one 128-token tile, run by the 128 threads
// that own its rows (thread r = token tile*128 + r, lane = r % 32); sync()
// is a barrier over exactly those threads. scratch holds FuseCfg<EW>::kScratch
// bytes. v = the row's logits before the bias; bias_r and noise_r are the
// additive terms already fetched.
template <int EW, class Sync>
__device__ __forceinline__ void select_and_aux(const RouterTcArgs& a, const float (&v)[EW],
                                               const float (&bias_r)[EW],
                                               const float (&noise_r)[EW], int tile, bool ok,
                                               int r, uint8_t* scratch, Sync sync) {
  using F = FuseCfg<EW>;
  const int E = a.E;
  const int lane = r & 31, wq = r >> 5;
  const int t = tile * 128 + r;
  float* red = reinterpret_cast<float*>(scratch);                // [128][kStride]
  float* pm = red + 128 * F::kStride;                            // [128][kStride]
  uint32_t* selm = reinterpret_cast<uint32_t*>(pm + 128 * F::kStride);  // [128]
  float* part_ps = reinterpret_cast<float*>(selm + 128);         // [kTcThreads]
  int* part_cs = reinterpret_cast<int*>(part_ps + kTcThreads);   // [kTcThreads]
  __shared__ int last_s;
  const bool valid = ok && t < a.T;
  float lg[EW], p[EW];
  float m = -INFINITY;
#pragma unroll
  for (int e = 0; e < EW; ++e) {
    lg[e] = e < E ? v[e] + bias_r[e] : -INFINITY;
    if (a.noise != nullptr && e < E && t < a.T) lg[e] += noise_r[e];
    m = fmaxf(m, lg[e]);
  }
  float ssum = 0.f;
#pragma unroll
  for (int e = 0; e < EW; ++e) {
    p[e] = e < E ? expf((lg[e] - m) * a.inv_tau) : 0.f;
    ssum += p[e];
  }
#pragma unroll
  for (int e = 0; e < EW; ++e) p[e] = p[e] / ssum;
  if (valid) {
#pragma unroll
    for (int e = 0; e < EW; ++e) {
      if (e < E && a.logits != nullptr) a.logits[static_cast<size_t>(t) * E + e] = lg[e];
      if (e < E && a.probs != nullptr) a.probs[static_cast<size_t>(t) * E + e] = p[e];
    }
  }
  uint32_t taken = 0;
  int sel_e[8];
  float sel_p[8];
  float wsum = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    sel_e[j] = 0;
    sel_p[j] = 0.f;
    if (j < a.k) {
      float bv = -INFINITY, bp = 0.f;
      int be = 0x7fffffff;
#pragma unroll
      for (int e = 0; e < EW; ++e)
        if (e < E && !((taken >> e) & 1u) && better(lg[e], e, bv, be)) { bv = lg[e]; be = e; bp = p[e]; }
      if (be >= E) {  // no finite logit left
        if (valid) set_error(a.ctl, MOE_DEVERR_EXPERT_RANGE);
        be = 0;
        bp = p[0];
      }
      taken |= 1u << be;
      sel_e[j] = be;
      sel_p[j] = bp;
      wsum += bp;
    }
  }
  if (valid) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < a.k) {
        a.idx[static_cast<size_t>(t) * a.k + j] = sel_e[j];
        a.w[static_cast<size_t>(t) * a.k + j] = sel_p[j] / wsum;
      }
  }
  // ---- z-loss partial of this tile: lse^2 per token, a fixed butterfly per
  // warp, then the 4 warps in order.
  __shared__ float zw_s[kTcThreads / 32];
  __shared__ double zd_s[kTcThreads];
  if (a.part_z != nullptr) {
    const float lse = m * a.inv_tau + logf(ssum);  // of the logits the softmax sees, l / tau
    float zt = valid ? lse * lse : 0.f;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) zt += __shfl_xor_sync(kFull, zt, off);
    if (lane == 0) zw_s[wq] = zt;
  }
  // ---- aux partials of this tile: thread (e, part) adds rows part, part +
  // kParts, ... of expert e; then the kParts sums are added in part order.
#pragma unroll
  for (int e = 0; e < EW; ++e) pm[r * F::kStride + e] = valid ? p[e] : 0.f;
  selm[r] = valid ? taken : 0u;
  sync();
  {
    const int e = r % EW, part = r / EW;
    float ps = 0.f;
    int cs = 0;
    for (int q = part; q < 128; q += F::kParts) {
      ps += pm[q * F::kStride + e];
      cs += (selm[q] >> e) & 1u;
    }
    part_ps[r] = ps;
    part_cs[r] = cs;
  }
  sync();
  if (r < E) {
    float ps = 0.f;
    int cs = 0;
    for (int q = 0; q < F::kParts; ++q) {
      ps += part_ps[q * EW + r];
      cs += part_cs[q * EW + r];
    }
    a.part_p[static_cast<size_t>(r) * a.ldb + tile] = ps;
    a.part_c[static_cast<size_t>(r) * a.ldb + tile] = cs;
  }
  if (a.part_z != nullptr && r == 0)
    a.part_z[tile] = ((zw_s[0] + zw_s[1]) + zw_s[2]) + zw_s[3];
  sync();
  if (r == 0) {
    __threadfence();
    last_s = atomicAdd(&a.ctl->route_ticket, 1u) == static_cast<unsigned>(a.ntile - 1);
  }
  sync();
  if (!last_s) return;
  __threadfence();
  // ---- last tile: thread (e, part) adds tiles part, part + kParts, ... in
  // float64, then thread e adds the kParts sums in part order.
  double* dps = reinterpret_cast<double*>(red);              // [kTcThreads]
  long long* dcs = reinterpret_cast<long long*>(dps + kTcThreads);  // [kTcThreads]
  {
    const int e = r % EW, part = r / EW;
    double ps = 0.0;
    long long cs = 0;
    if (e < E)
      for (int b = part; b < a.ntile; b += F::kParts) {
        ps += static_cast<double>(__ldcg(a.part_p + static_cast<size_t>(e) * a.ldb + b));
        cs += __ldcg(a.part_c + static_cast<size_t>(e) * a.ldb + b);
      }
    dps[r] = ps;
    dcs[r] = cs;
  }
  sync();
  // thread e: its expert's term f_e * P_e; thread 0 adds the terms in expert order
  __shared__ double term_s[kFuseMaxE];
  if (r < E) {
    double ps = 0.0;
    long long cs = 0;
    for (int q = 0; q < F::kParts; ++q) {
      ps += dps[q * EW + r];
      cs += dcs[q * EW + r];
    }
    term_s[r] = (static_cast<double>(cs) / (static_cast<double>(a.T) * a.k)) * (ps / a.T);
  }
  sync();
  if (r == 0) {
    double tot = 0.0;
    for (int e = 0; e < E; ++e) tot += term_s[e];
    *a.aux = static_cast<float>(E * tot);
  }
  if (a.part_z != nullptr) {  // z-loss: tiles r, r + 128, ... then a fixed tree, / T
    double zs = 0.0;
    for (int b = r; b < a.ntile; b += kTcThreads) zs += static_cast<double>(__ldcg(a.part_z + b));
    zd_s[r] = zs;
    sync();
    for (int st = kTcThreads / 2; st > 0; st >>= 1) {
      if (r < st) zd_s[r] += zd_s[r + st];
      sync();
    }
    if (r == 0) *a.z_out = static_cast<float>(zd_s[0] / a.T);
  }
  if (r == 0) a.ctl->route_ticket = 0u;
}

// kFuseE = 0: partial logits out (router_select follows); 8, 16 or 32: the
// fused selection above with that width.
template <bool kTmaB, int kFuseE>
__global__ void __launch_bounds__(kTcThreads, 1)
router_tc(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
          RouterTcArgs a) {
  pdl_begin();
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kTcStages], empty_bar[kTcStages], done_bar;
  __shared__ uint32_t tmem_base_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int tile = blockIdx.x / a.KS;
  const int ks = blockIdx.x - tile * a.KS;
  const int nkb = a.dk / 64;
  const int b_boxes = kTmaB ? a.Epad / 64 : 0;
  const uint32_t a_bytes = 128 * 128, stage_bytes = a_bytes + b_boxes * 8192;
  const int nst = a.stages;
  uint8_t* ring = smem;
  uint8_t* wgt = smem + nst * stage_bytes;  // staged Wg^T (E <= 32)
  // k-block kb's E real rows start at kb * E * 128 bytes (E is a multiple of
  // 8, so every block starts on a 1024-byte swizzle atom). The MMA's N = Epad
  // also reads rows E..Epad-1 (at most one 8-row atom): the next block's first
  // rows, or the 1 KB of slack after the last block. They land only in
  // accumulator columns E..Epad-1, which nothing reads.
  const uint32_t wgt_kb_bytes = static_cast<uint32_t>(a.E) * 128;
  // Accumulator slots: k-block kb accumulates into TMEM columns
  // [(kb / G) * Epad, +Epad), G k-blocks per slot, as many slots as 512
  // columns hold. The epilogue adds the slots in IEEE fp32, so a tensor-core
  // accumulation chain is at most 4*G MMAs long.
  const int nslot_cap = a.tmem_cap / a.Epad;
  const int G = (nkb + nslot_cap - 1) / nslot_cap;
  const int nslot = (nkb + G - 1) / G;
  uint32_t tcols = 32;
  while (tcols < static_cast<uint32_t>(nslot * a.Epad)) tcols <<= 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < nst; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
    mbar_init(&done_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_s, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;

  // Wg^T for this CTA's d-range (staged path) as K-major 128-byte-swizzled
  // rows: expert e, k-block kb -> row e of block kb, 16-byte chunk
  // (kk/8) ^ (e%8). A task is 8 consecutive d-rows x 8 experts: eight 16-byte
  // loads (one Wg row slice each), an 8x8 transpose of bf16 pairs with byte
  // permutes, eight 16-byte stores (one expert's 8 k-values each). Tasks of
  // the real experts come first; experts E..Epad-1 are zero. Each thread's
  // first loads go out before the x tiles' TMA loads, so they do not queue
  // behind them. Only the real experts' rows are staged (see wgt_kb_bytes).
  const int k0 = ks * a.dk;
  const int nchunk = a.dk / 8, groups = a.E / 8;
  const int ntask = kTmaB ? 0 : nchunk * groups;
  auto load_task = [&](int i, uint32_t (&in)[8][4]) {
    const int g = i / nchunk, ch = i - g * nchunk;
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(a.wg + static_cast<size_t>(k0 + ch * 8 + rr) * a.E) + g);
      in[rr][0] = u.x;
      in[rr][1] = u.y;
      in[rr][2] = u.z;
      in[rr][3] = u.w;
    }
  };
  auto store_task = [&](int i, const uint32_t (&in)[8][4]) {
    const int g = i / nchunk, ch = i - g * nchunk;
    const int kb = ch >> 3, c = ch & 7;
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int e = g * 8 + jj;
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)  // k-values 2q (low half) and 2q+1 (high half)
        o[q] = __byte_perm(in[2 * q][jj >> 1], in[2 * q + 1][jj >> 1], (jj & 1) ? 0x7632 : 0x5410);
      const uint32_t off = kb * wgt_kb_bytes + e * 128 + (((c ^ e) & 7) << 4);
      *reinterpret_cast<uint4*>(wgt + off) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  };
  uint32_t in0[8][4];
  if (static_cast<int>(threadIdx.x) < ntask) load_task(threadIdx.x, in0);

  // The first ring stages are free: start their loads now.
  const int pre = nkb < nst ? nkb : nst;
  auto issue = [&](int kb, int st) {
    uint8_t* sa = ring + st * stage_bytes;
    const int kx = ks * a.dk + kb * 64;
    mbar_arrive_expect_tx(&full_bar[st], stage_bytes);
    tma_load_2d(sa, &tmX, &full_bar[st], kx, tile * 128);
    for (int j = 0; j < b_boxes; ++j) tma_load_2d(sa + a_bytes + j * 8192, &tmW, &full_bar[st], j * 64, kx);
  };
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmX);
    if (kTmaB) prefetch_tmap(&tmW);
    for (int kb = 0; kb < pre; ++kb) issue(kb, kb);
  }
  if (!kTmaB) {
    // the next task's loads go out before this task's stores
    for (int i = threadIdx.x; i < ntask; i += kTcThreads) {
      uint32_t nxt[8][4];
      const bool more = i + kTcThreads < ntask;
      if (more) load_task(i + kTcThreads, nxt);
      store_task(i, in0);
      if (more) {
#pragma unroll
        for (int rr = 0; rr < 8; ++rr)
#pragma unroll
          for (int q = 0; q < 4; ++q) in0[rr][q] = nxt[rr][q];
      }
    }
    fence_proxy_async_smem();  // generic-proxy writes, read by the tensor core
    __syncthreads();
  }

  // The fused selection's additive terms, fetched while the MMAs run.
  constexpr int kEW = kFuseE > 0 ? kFuseE : 1;
  float bias_r[kEW], noise_r[kEW];
#pragma unroll
  for (int e = 0; e < kEW; ++e) {
    bias_r[e] = 0.f;
    noise_r[e] = 0.f;
  }
  if constexpr (kFuseE != 0) {
    const int t = tile * 128 + warp * 32 + lane;
    if (ks == 0) {
#pragma unroll
      for (int e = 0; e < kEW; ++e) {
        if (e < a.E && a.bias != nullptr) bias_r[e] = __ldg(a.bias + e);
        if (e < a.E && a.noise != nullptr && t < a.T) noise_r[e] = __ldg(a.noise + static_cast<size_t>(t) * a.E + e);
      }
    }
  }
  bool ok = true;
  if (warp == 0 && lane == 0) {
    uint32_t phase = 1;  // the prologue filled round 0
    int st = pre % nst;
    if (pre < nst) phase = 0;
    int kb = pre;
    for (; kb < nkb; ++kb) {
      if (!mbar_wait_bounded(&empty_bar[st], phase ^ 1u)) { set_error(a.ctl, MOE_DEVERR_TIMEOUT); break; }
      issue(kb, st);
      if (++st == nst) { st = 0; phase ^= 1u; }
    }
    if (kb < nkb) {
      // stopped early: wait (bounded) for the last load issued into each
      // stage, so that none lands after the block has gone
      for (int s2 = 0; s2 < nst && s2 < kb; ++s2) {
        const int last = s2 + ((kb - 1 - s2) / nst) * nst;
        (void)mbar_wait_bounded(&full_bar[s2], static_cast<uint32_t>(last / nst) & 1u);
      }
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = make_idesc_bf16(128, a.Epad, !kTmaB);
    uint32_t phase = 0;
    bool issued = false;
    for (int kb = 0, st = 0; kb < nkb; ++kb) {
      if (!mbar_wait_bounded(&full_bar[st], phase)) { set_error(a.ctl, MOE_DEVERR_TIMEOUT); break; }
      tc_fence_after();
      const uint32_t a_addr = smem_u32(ring + st * stage_bytes);
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>((kb / G) * a.Epad);
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t adesc = make_sw128_desc(a_addr + kk * 32, 16, 1024);
        const uint64_t bdesc = kTmaB ? make_sw128_desc(a_addr + a_bytes + kk * 2048, 8192, 1024)
                                     : make_sw128_desc(smem_u32(wgt) + kb * wgt_kb_bytes + kk * 32, 16, 1024);
        umma_bf16(d_tmem, adesc, bdesc, idesc, ((kb % G) | kk) != 0 ? 1u : 0u);
      }
      issued = true;
      umma_commit(&empty_bar[st]);
      if (++st == nst) { st = 0; phase ^= 1u; }
    }
    if (issued) umma_commit(&done_bar);
    else mbar_arrive(&done_bar);
  }
  {
    int d_ok = 0;
    if (lane == 0) d_ok = mbar_wait_bounded(&done_bar, 0);
    d_ok = __shfl_sync(kFull, d_ok, 0);
    if (!d_ok) { if (lane == 0) set_error(a.ctl, MOE_DEVERR_TIMEOUT); ok = false; }
  }
  tc_fence_after();
  if constexpr (kFuseE == 0) {
    // ---- accumulator rows -> partial logits [ks][t][e]
    {
      const int r = warp * 32 + lane;
      const int t = tile * 128 + r;
      float* dst = a.partial + static_cast<size_t>(ks) * a.T * a.E + static_cast<size_t>(t) * a.E;
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
      for (int c0 = 0; c0 < a.Epad; c0 += 16) {
        float sum[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) sum[i] = 0.f;
        for (int sl = 0; sl < nslot; ++sl) {  // slot order
          uint32_t u[16];
          tmem_ld_32x32b_x16(trow + sl * a.Epad + c0, u);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) sum[i] += __uint_as_float(u[i]);
        }
        uint32_t v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(sum[i]);
        if (t < a.T && ok) {
          if (c0 + 16 <= a.E) {
#pragma unroll
            for (int i = 0; i < 16; i += 4)
              *reinterpret_cast<float4*>(dst + c0 + i) =
                  make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                              __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (c0 + i < a.E) dst[c0 + i] = __uint_as_float(v[i]);
          }
        }
      }
    }
  } else {
    // The ring is idle (every MMA has completed): it holds the row buffers.
    const int r = warp * 32 + lane;
    float v[kEW];
    slot_sums<kEW>(tmem_base + (static_cast<uint32_t>(warp * 32) << 16), nslot, a.Epad, v);
    if (a.KS > 1) cluster_row_sums<kEW>(a.KS, ks, r, reinterpret_cast<float*>(smem), v);
    if (ks == 0) select_and_aux<kEW>(a, v, bias_r, noise_r, tile, ok, r, smem, [] { __syncthreads(); });
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tcols);
  }
}

// Persistent fused router, d unsplit (KS = 1), for more token tiles than
// SMs: one CTA per SM walks the tiles blockIdx.x, blockIdx.x + gridDim.x, ...
// Six warps: warp 0 (one thread) streams x k-blocks of all its tiles through
// the ring, warp 1 (one thread) issues the MMAs of tile j into accumulator
// j % 2 (two of 256 tensor-memory columns), warps 2-5 (thread = token row;
// warp w reads lane quarter w % 4) run the selection and aux partials of tile
// j while tile j + 1 loads and multiplies. Same arithmetic as router_tc's
// fused path with KS = 1.
// Wg is not staged: each stage also carries its k-blocks' Wg rows, TMA-loaded
// as E/8 boxes of 8 experts x 64 rows (1 KB each, no swizzle, packed E/8 KB
// per k-block) that the MMA reads as its MN-major operand (8-row core
// matrices 16 bytes wide, 128 bytes apart along K, 1 KB apart along N). An
// MMA of N = Epad > E also reads the (Epad - E)/8 KB after its k-block's
// boxes (the next k-block's, or the 1 KB of slack after the ring) into
// accumulator columns that nothing reads. Without the 64 KB of staged Wg^T
// (d = 4096, E = 8) the ring holds a third 64 KB stage, and the stream runs
// with more bytes in flight per SM.
constexpr int kPersistThreads = 192;
constexpr int kPersistAccCols = 256;

__device__ __forceinline__ void epi_bar_sync() {  // the four selection warps
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

template <int EW>
__global__ void __launch_bounds__(kPersistThreads, 1)
router_tc_persist(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                  RouterTcArgs a) {
  pdl_begin();
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kTcStages], empty_bar[kTcStages];
  __shared__ __align__(8) uint64_t tfull_bar[2], tempty_bar[2], done_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int okw_s[4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int nkb = a.d / 64;
  constexpr uint32_t kBoxBytes = 128 * 128;  // one k-block of 128 token rows
  const int sub = a.sub;                     // k-blocks per stage (divides nkb)
  const int nkg = nkb / sub;                 // stage loads per tile
  const uint32_t wkb_bytes = static_cast<uint32_t>(a.E / 8) * 1024;  // one k-block's Wg boxes
  const uint32_t xs_bytes = kBoxBytes * sub;
  const uint32_t stage_bytes = xs_bytes + wkb_bytes * sub;           // a multiple of 1024
  const int nst = a.stages;
  uint8_t* ring = smem;
  uint8_t* scratch = smem + nst * stage_bytes + 1024;  // after 1 KB of slack
  const int nslot_cap = kPersistAccCols / a.Epad;
  const int G = (nkb + nslot_cap - 1) / nslot_cap;  // k-blocks per accumulator slot
  const int nslot = (nkb + G - 1) / G;
  const int my_tiles = static_cast<int>(blockIdx.x) < a.ntile
                           ? (a.ntile - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                           : 0;
  const int total = my_tiles * nkg;  // ring loads of this CTA
  const int pre = total < nst ? total : nst;

  // load i: tile i / nkg, k-blocks sub * (i % nkg) + [0, sub), stage i % nst;
  // the sub boxes of a row's consecutive 128-byte pieces go out together
  auto issue = [&](int i) {
    const int j = i / nkg, kg = i - j * nkg, st = i % nst;
    const int tile = static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x);
    uint8_t* sa = ring + st * stage_bytes;
    mbar_arrive_expect_tx(&full_bar[st], stage_bytes);
    for (int u = 0; u < sub; ++u)
      tma_load_2d(sa + u * kBoxBytes, &tmX, &full_bar[st], (kg * sub + u) * 64, tile * 128);
    for (int u = 0; u < sub; ++u)
      for (int n8 = 0; n8 < a.E / 8; ++n8)
        tma_load_2d(sa + xs_bytes + u * wkb_bytes + n8 * 1024, &tmW, &full_bar[st], n8 * 8,
                    (kg * sub + u) * 64);
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < nst; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&tfull_bar[b], 1); mbar_init(&tempty_bar[b], 4); }
    mbar_init(&done_bar, 1);
    fence_mbar_init();
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmW);
    for (int i = 0; i < pre; ++i) issue(i);  // the ring's first round
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_s, 2 * kPersistAccCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;

  if (warp == 0) {
    if (lane == 0) {
      int i = pre;
      for (; i < total; ++i) {
        const int st = i % nst, round = i / nst;
        if (!mbar_wait_bounded(&empty_bar[st], (round & 1) ^ 1u)) {
          set_error(a.ctl, MOE_DEVERR_TIMEOUT);
          break;
        }
        issue(i);
      }
      // wait (bounded) for the last load issued into each stage to land
      for (int st = 0; st < nst && st < i; ++st) {
        const int last = st + ((i - 1 - st) / nst) * nst;
        mbar_wait_bounded(&full_bar[st], static_cast<uint32_t>(last / nst) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc_bf16(128, a.Epad, false);  // Wg rows: MN-major
      bool issued = false, ok = true;
      int i = 0;
      for (int j = 0; j < my_tiles && ok; ++j) {
        const int acc = j & 1;
        if (!mbar_wait_bounded(&tempty_bar[acc], static_cast<uint32_t>((j >> 1) & 1) ^ 1u)) {
          set_error(a.ctl, MOE_DEVERR_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t dbase = tmem_base + static_cast<uint32_t>(acc * kPersistAccCols);
        for (int kg = 0; kg < nkg; ++kg, ++i) {
          const int st = i % nst;
          if (!mbar_wait_bounded(&full_bar[st], static_cast<uint32_t>(i / nst) & 1u)) {
            set_error(a.ctl, MOE_DEVERR_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t s_addr = smem_u32(ring + st * stage_bytes);
          for (int u = 0; u < sub; ++u) {
            const int kb = kg * sub + u;
            const uint32_t a_addr = s_addr + u * kBoxBytes;
            const uint32_t b_addr = s_addr + xs_bytes + u * wkb_bytes;
            const uint32_t d_tmem = dbase + static_cast<uint32_t>((kb / G) * a.Epad);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t adesc = make_sw128_desc(a_addr + kk * 32, 16, 1024);
              const uint64_t bdesc = make_noswz_desc(b_addr + kk * 256, 128, 1024);
              umma_bf16(d_tmem, adesc, bdesc, idesc, ((kb % G) | kk) != 0 ? 1u : 0u);
            }
          }
          issued = true;
          umma_commit(&empty_bar[st]);
        }
        if (ok) umma_commit(&tfull_bar[acc]);
      }
      // every MMA issued has completed before the tensor memory is freed
      if (issued) {
        umma_commit(&done_bar);
        mbar_wait_bounded(&done_bar, 0);
      }
    }
  } else {
    const int q = warp & 3;  // the lane quarter this warp may read
    const int r = q * 32 + lane;
    float bias_r[EW], noise_r[EW];
#pragma unroll
    for (int e = 0; e < EW; ++e) {
      bias_r[e] = (e < a.E && a.bias != nullptr) ? __ldg(a.bias + e) : 0.f;
      noise_r[e] = 0.f;
    }
    for (int j = 0; j < my_tiles; ++j) {
      const int acc = j & 1;
      const int tile = static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x);
      const int t = tile * 128 + r;
      if (a.noise != nullptr && t < a.T) {
#pragma unroll
        for (int e = 0; e < EW; ++e)
          if (e < a.E) noise_r[e] = __ldg(a.noise + static_cast<size_t>(t) * a.E + e);
      }
      int okw = 1;
      if (lane == 0) okw = mbar_wait_bounded(&tfull_bar[acc], static_cast<uint32_t>(j >> 1) & 1u);
      okw = __shfl_sync(kFull, okw, 0);
      if (lane == 0) okw_s[q] = okw;
      epi_bar_sync();
      if (!(okw_s[0] && okw_s[1] && okw_s[2] && okw_s[3])) {  // the four warps leave together
        if (r == 0) set_error(a.ctl, MOE_DEVERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      float v[EW];
      slot_sums<EW>(tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                        static_cast<uint32_t>(acc * kPersistAccCols),
                    nslot, a.Epad, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[acc]);  // accumulator free for tile j + 2
      select_and_aux<EW>(a, v, bias_r, noise_r, tile, true, r, scratch, [] { epi_bar_sync(); });
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * kPersistAccCols);
  }
}

bool use_fused(int d, int E, moe_dtype_t dt) {
  const size_t bytes = static_cast<size_t>((d + 7) / 8) * 256;  // fp32 pairs, 256 B per 8 rows
  return dt == MOE_F32 && E <= 8 && d % 8 == 0 && bytes <= 160 * 1024;
}

size_t fused_smem_bytes(int d) { return static_cast<size_t>((d + 7) / 8) * 256; }

// Tensor-core router plan: split factor KS (a power of two <= 8 dividing the
// d/64 k-blocks) grows while the grid stays within the SMs; the staged Wg^T
// of one CTA must fit in 128 KB; the ring takes what is left of 227 KB, up to
// kTcStages stages.
// Split over d: the grid may reach kTcFill x (SMs / 2) CTAs. The unfused
// path keeps it at half the SMs (more splits cost router_select more partial
// traffic than they save); the fused path, whose split is reduced on chip,
// goes to two CTAs per SM with a 4-stage ring each (measured fastest).
constexpr int kTcFill = 1;
constexpr int kTcFillFused = 2;
constexpr int kTcStagesFused = 4;

struct TcPlan {
  bool use = false;
  bool tma_b = false;
  int fuse_e = 0;  // 8, 16 or 32: router_tc<false, fuse_e> selects and reduces the aux loss too
  int Epad = 0, KS = 1, ntile = 0, stages = 0;
  size_t smem = 0;
  size_t stage = 0, scratch = 0;  // bytes of one ring stage; the fused selection's row buffers
};

TcPlan plan_tc(int T, int d, int E, moe_dtype_t dt) {
  TcPlan p;
  if (dt != MOE_BF16 || T <= 0 || d % 64 != 0) return p;
  if (E % 64 == 0) {
    p.tma_b = true;
    p.Epad = E;
  } else if (E <= 32 && E % 8 == 0) {
    p.Epad = (E + 15) / 16 * 16;
  } else {
    return p;
  }
  p.ntile = (T + 127) / 128;
  const int nkb = d / 64;
  const bool fusable = !p.tma_b && E <= kFuseMaxE;
  const int fill = fusable ? kTcFillFused : kTcFill;
  int ks = 1;
  while (ks < kMaxKS && p.ntile * ks * 2 <= num_sms() * fill && nkb % (ks * 2) == 0) ks *= 2;
  if (!p.tma_b)
    while (static_cast<size_t>(d / ks) * E * 2 > 128 * 1024 && ks < kMaxKS && nkb % (ks * 2) == 0) ks *= 2;
  if (!p.tma_b && static_cast<size_t>(d / ks) * E * 2 > 128 * 1024) return p;
  p.KS = ks;
  const size_t stage = 128 * 128 + (p.tma_b ? static_cast<size_t>(p.Epad / 64) * 8192 : 0);
  // staged Wg^T: the real rows, plus one atom of slack read as padding rows
  const size_t wgt = p.tma_b ? 0 : static_cast<size_t>(d / ks) * E * 2 + (p.Epad != E ? 1024 : 0);
  const size_t avail = 227 * 1024 - 1024 - wgt;
  p.stages = static_cast<int>(std::min<size_t>(fusable ? kTcStagesFused : kTcStages, avail / stage));
  if (p.stages < 2) return p;
  p.smem = 1024 + p.stages * stage + wgt;
  p.stage = stage;
  p.use = true;
  // The fused selection reuses the ring for its row buffers.
  if (fusable) {
    const int ew = E <= 8 ? 8 : (E <= 16 ? 16 : 32);
    const size_t scratch = ew == 8 ? FuseCfg<8>::kScratch
                         : ew == 16 ? FuseCfg<16>::kScratch : FuseCfg<32>::kScratch;
    if (p.stages * stage >= scratch) {
      p.fuse_e = ew;
      p.scratch = scratch;
    }
  }
  return p;
}

}  // namespace

static int route_max_blocks(int T) {
  return std::max(std::max(1, (T + kSelectTokensPerBlock - 1) / kSelectTokensPerBlock), num_sms());
}

size_t route_partials_bytes(int T, int E) {
  // per-block sums then counts (expert-major), the per-expert terms, the
  // per-block z-loss sums
  return align_up(static_cast<size_t>(route_max_blocks(T)) * E * 4) * 2 + align_up(256 * 8) +
         align_up(static_cast<size_t>(route_max_blocks(T)) * 4);  // z-loss partials
}

size_t route_logits_scratch_bytes(int T, int d, int E) {
  (void)d;
  return align_up(static_cast<size_t>(kMaxKS) * T * E * 4);
}

cudaError_t launch_route(const void* x, const void* wg, const float* bias, const float* noise,
                         moe_dtype_t dt, int T, int d, int E, int k, int32_t* idx, float* w,
                         float* aux, float* z_out, float* logits, float* probs,
                         float* logits_scratch, void* partials, Control* ctl, cudaStream_t s,
                         float temperature, AuxJob* defer_aux) {
  const float inv_tau = 1.0f / temperature;
  const int ldb = route_max_blocks(T);
  float* part_p = static_cast<float*>(partials);
  int32_t* part_c = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(partials) +
                                               align_up(static_cast<size_t>(ldb) * E * 4));
  double* terms = reinterpret_cast<double*>(static_cast<uint8_t*>(partials) +
                                            2 * align_up(static_cast<size_t>(ldb) * E * 4));
  float* part_z = z_out == nullptr ? nullptr
                                   : reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(terms) +
                                                              align_up(256 * 8));
  int nblk = 0;
  // With defer_aux the loss's last step is described for a later kernel
  // instead of being run here.
  // Only the paths that would launch aux_reduce defer (the fused tensor-core
  // router's own last-tile step costs less than a later kernel's).
  auto defer = [&](int blocks) {
    *defer_aux = AuxJob{1, part_p, part_c, part_z, terms, aux, z_out, ldb, blocks, E, T, k};
  };
  if (defer_aux != nullptr) defer_aux->pending = 0;
  // The fp32 E <= 8 kernel has neither the noise input, the z-loss nor a temperature.
  if (use_fused(d, E, dt) && noise == nullptr && z_out == nullptr && inv_tau == 1.0f) {
    const int groups = (T + kFusedTokensPerGroup - 1) / kFusedTokensPerGroup;
    const int grid = std::max(1, std::min(groups, num_sms()));
    const size_t smem = fused_smem_bytes(d);
    auto kern = router_fused_e8<float>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(kFusedThreads), smem, s, false,
                                     static_cast<const float*>(x), static_cast<const float*>(wg),
                                     bias, T, d, E, k, idx, w, logits, probs, part_p, part_c, ldb,
                                     ctl);
    if (e != cudaSuccess) return e;
    nblk = grid;
  } else {
    int KS = 1;
    const TcPlan tp = plan_tc(T, d, E, dt);
    if (tp.use) {
      CUtensorMap tx, tw;
      if (!make_tma_2d_bf16(&tx, x, static_cast<uint64_t>(T), d, 128)) return cudaErrorInvalidValue;
      if (tp.tma_b) {
        if (!make_tma_2d_bf16(&tw, wg, static_cast<uint64_t>(d), E, 64)) return cudaErrorInvalidValue;
      } else {
        tw = tx;  // unused by the staged path
      }
      RouterTcArgs a = {};
      a.T = T; a.d = d; a.E = E; a.Epad = tp.Epad; a.KS = tp.KS; a.dk = d / tp.KS;
      a.stages = tp.stages;
      a.tmem_cap = 512;
      a.inv_tau = inv_tau;
      a.wg = static_cast<const __nv_bfloat16*>(wg);
      a.partial = logits_scratch;
      a.ctl = ctl;
      const dim3 grid(tp.ntile * tp.KS);
      if (tp.fuse_e != 0) {
        // one kernel: gate GEMM, cluster reduction over d, selection, aux loss
        a.bias = bias; a.k = k; a.ntile = tp.ntile; a.ldb = ldb;
        a.idx = idx; a.w = w; a.logits = logits; a.probs = probs;
        a.part_p = part_p; a.part_c = part_c; a.aux = aux;
        a.noise = noise; a.part_z = part_z; a.z_out = z_out;
        if (tp.KS == 1 && tp.ntile > num_sms()) {
          // persistent: one CTA per SM walks the tiles
          const size_t fixed = 1024 + 1024 + tp.scratch;  // alignment, slack, selection buffers
          const size_t budget = 227 * 1024 - 2048;  // dynamic shared memory next to the static
          // k-blocks per stage: 4 (each token row's 512 consecutive bytes requested
          // together, measured 14-20% faster than one k-block per stage at T =
          // 32768-65536), fewer if two such stages do not fit
          const size_t kbytes = 16384 + static_cast<size_t>(E / 8) * 1024;  // x and Wg of one k-block
          int sub = 4;
          while (sub > 1 && ((d / 64) % sub != 0 || fixed + 2 * kbytes * static_cast<size_t>(sub) > budget)) sub >>= 1;
          const size_t sbytes = kbytes * static_cast<size_t>(sub);
          CUtensorMap tw2;
          const int st = fixed + 2 * sbytes <= budget
                             ? static_cast<int>(std::min<size_t>(kTcStages, (budget - fixed) / sbytes))
                             : 0;
          if (st >= 2 && (reinterpret_cast<uintptr_t>(wg) & 15u) == 0 &&
              make_tma_2d_bf16_plain(&tw2, wg, static_cast<uint64_t>(d), E, 8, 64)) {
            // at least 120 KB, so that no two CTAs share an SM (each takes all
            // 512 tensor-memory columns)
            const size_t smem = std::max<size_t>(fixed + static_cast<size_t>(st) * sbytes, 120 * 1024);
            a.stages = st;
            a.sub = sub;
            auto pk = tp.fuse_e == 8 ? router_tc_persist<8>
                    : tp.fuse_e == 16 ? router_tc_persist<16> : router_tc_persist<32>;
            cudaFuncSetAttribute(pk, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
            return launch_pdl(pk, dim3(std::min(tp.ntile, num_sms())), dim3(kPersistThreads), smem, s,
                              false, tx, tw2, a);
          }
        }
        auto kern = tp.fuse_e == 8 ? router_tc<false, 8>
                  : tp.fuse_e == 16 ? router_tc<false, 16> : router_tc<false, 32>;
        // More CTAs than SMs: take ring stages away while that lets the whole
        // grid be resident at once (each CTA stages Wg^T once, no second wave).
        size_t smem = tp.smem;
        const long long G = grid.x, sms = num_sms();
        int nb = 1;
        if (G > sms) {
          for (int st = tp.stages; st >= 2 && static_cast<size_t>(st) * tp.stage >= tp.scratch; --st) {
            const size_t sm = tp.smem - static_cast<size_t>(tp.stages - st) * tp.stage;
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
            int n = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kTcThreads, sm) != cudaSuccess) {
              cudaGetLastError();
              break;
            }
            if (st == tp.stages) nb = std::max(n, 1);
            if (static_cast<long long>(n) * sms >= G) {
              a.stages = st;
              smem = sm;
              nb = n;
              break;
            }
          }
        }
        // CTAs that share an SM split its 512 tensor-memory columns.
        const long long per_sm = std::min<long long>(nb, (G + sms - 1) / sms);
        while (a.tmem_cap > tp.Epad && a.tmem_cap * per_sm > 512) a.tmem_cap >>= 1;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        return launch_pdl_cluster(kern, grid, dim3(kTcThreads), smem, s, tp.KS, tx, tw, a);
      }
      auto kern = tp.tma_b ? router_tc<true, 0> : router_tc<false, 0>;
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(tp.smem));
      const cudaError_t e = launch_pdl(kern, grid, dim3(kTcThreads), tp.smem, s, false, tx, tw, a);
      if (e != cudaSuccess) return e;
      KS = tp.KS;
    } else if (T > 0) {
      dim3 g1((T + 63) / 64, (E + 63) / 64);
      const cudaError_t e =
          dt == MOE_BF16
              ? launch_pdl(router_gemm_tiled<__nv_bfloat16>, g1, dim3(256), 0, s, false,
                           static_cast<const __nv_bfloat16*>(x),
                           static_cast<const __nv_bfloat16*>(wg), T, d, E, logits_scratch)
              : launch_pdl(router_gemm_tiled<float>, g1, dim3(256), 0, s, false,
                           static_cast<const float*>(x), static_cast<const float*>(wg), T, d, E,
                           logits_scratch);
      if (e != cudaSuccess) return e;
    }
    const int g2 = std::max(1, (T + kSelectTokensPerBlock - 1) / kSelectTokensPerBlock);
    const int epl = (E + 31) / 32;
    auto sel = epl <= 1 ? router_select<1>
             : epl <= 2 ? router_select<2>
             : epl <= 4 ? router_select<4>
                        : router_select<8>;
    const cudaError_t e = launch_pdl(sel, dim3(g2), dim3(kSelectWarps * 32), 0, s, false,
                                     static_cast<const float*>(logits_scratch), KS, bias, noise, T,
                                     E, k, idx, w, logits, probs, part_p, part_c, part_z, ldb, inv_tau,
                                     ctl);
    if (e != cudaSuccess) return e;
    nblk = g2;
  }
  if (defer_aux != nullptr) {
    defer(nblk);
    return cudaSuccess;
  }
  return launch_pdl(aux_reduce, dim3(E), dim3(kAuxThreads), 0, s, false,
                    static_cast<const float*>(part_p), static_cast<const int32_t*>(part_c),
                    static_cast<const float*>(part_z), ldb, nblk, E, T, k, terms, aux, z_out, ctl);
}

}  // namespace moe
