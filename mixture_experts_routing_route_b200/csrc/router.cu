// Router: gate GEMM (fp32 accumulate), softmax over E, top-k by selection
// (ties to the lower expert index), renormalisation of the k weights, and the
// load-balance loss aux = E * sum_i f_i * P_i.
//
// Sources: "ops-transformer MoE operators" blog, 实现 (MoEGatingForward:
// Softmax, TopK by a selection rather than a sort, NormalizeWeights);
// "MoE Router" page (Linear(hidden, E, bias=False) -> softmax -> topk ->
// renormalise); "MegaBlocks 01", section 1 (bias-free linear router).
//
// Two paths:
//  * E <= 8 and Wg small enough for shared memory: one fused kernel. A warp
//    owns 4 tokens at a time; each lane streams 16-byte slices of the 4 x rows
//    and multiplies them with the staged Wg rows, a 31-shuffle reduce-scatter
//    leaves lane l with logit (token l/8, expert l%8), and selection then runs
//    inside 8-lane groups. x is read from HBM exactly once.
//  * otherwise: a tiled fp32 GEMM writes the logits [T, E] to scratch, then a
//    warp-per-token kernel does softmax / top-k / renormalisation.
// Both end with per-block aux partials reduced in a fixed order by the last
// block to finish (a ticket counter), so the loss is deterministic.
#include "common.cuh"
#include <cfloat>
#include <cmath>
#include <algorithm>

namespace moe {

namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ bool better(float va, int ea, float vb, int eb) {
  return va > vb || (va == vb && ea < eb);
}

// Reduce the aux partials of all blocks, then aux = E * sum_e f_e * P_e, in
// float64 and in a fixed order: expert e's partials are summed by one warp
// (lane l takes blocks l, l+32, ...; a butterfly combines the lanes) and the
// per-expert terms are added by a tree over 256 slots. The result does not
// depend on the block size. Run by every thread of the last block.
__device__ void finalize_aux(const float* part_p, const int32_t* part_c, int nblk, int E, int T,
                             int k, float* aux) {
  __shared__ double red[256];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int i = threadIdx.x; i < 256; i += blockDim.x) red[i] = 0.0;
  __syncthreads();
  for (int e = warp; e < E; e += nw) {
    double ps = 0.0;
    long long cs = 0;
    for (int b = lane; b < nblk; b += 32) {
      ps += static_cast<double>(__ldcg(part_p + static_cast<size_t>(b) * E + e));
      cs += __ldcg(part_c + static_cast<size_t>(b) * E + e);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      ps += __shfl_xor_sync(kFull, ps, off);
      cs += __shfl_xor_sync(kFull, cs, off);
    }
    if (lane == 0 && T > 0)
      red[e] = (static_cast<double>(cs) / (static_cast<double>(T) * k)) * (ps / T);
  }
  __syncthreads();
  for (int s = 128; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0 && aux) *aux = static_cast<float>(E * red[0]);
}

// Write this block's partials, take a ticket, and let the last block reduce.
__device__ void block_partials_and_ticket(const float* blk_p, const int32_t* blk_c, float* part_p,
                                          int32_t* part_c, int E, int T, int k, float* aux,
                                          Control* ctl) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    part_p[static_cast<size_t>(blockIdx.x) * E + e] = blk_p[e];
    part_c[static_cast<size_t>(blockIdx.x) * E + e] = blk_c[e];
  }
  __threadfence();
  __syncthreads();
  __shared__ bool is_last;
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(&ctl->route_ticket, 1u);
    is_last = (prev == gridDim.x - 1);
  }
  __syncthreads();
  if (is_last) {
    __threadfence();
    finalize_aux(part_p, part_c, gridDim.x, E, T, k, aux);
    if (threadIdx.x == 0) ctl->route_ticket = 0u;
  }
}

// ---------------------------------------------------------------- fused, E <= 8
template <typename Tin>
struct VecTraits;
template <> struct VecTraits<__nv_bfloat16> {
  static constexpr int kVec = 8;  // elements per 16-byte load
  static __device__ __forceinline__ void unpack(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};
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
                float* __restrict__ part_p, int32_t* __restrict__ part_c, float* __restrict__ aux,
                Control* ctl) {
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
  block_partials_and_ticket(tot_p, tot_c, part_p, part_c, E, T, k, aux, ctl);
}

// ---------------------------------------------------------------- general path
// logits[T, E] = x[T, d] * Wg[d, E], 64x64 tiles, 256 threads with 4x4 each.
template <typename Tin>
__global__ void __launch_bounds__(256)
router_gemm_tiled(const Tin* __restrict__ x, const Tin* __restrict__ wg, int T, int d, int E,
                  float* __restrict__ out) {
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

// Warp per token: lane l holds experts l + 32q, q < EPL.
template <int EPL>
__global__ void __launch_bounds__(256)
router_select(const float* __restrict__ logits_in, const float* __restrict__ bias, int T, int E,
              int k, int32_t* __restrict__ idx_out, float* __restrict__ w_out,
              float* __restrict__ logits_out, float* __restrict__ probs_out,
              float* __restrict__ part_p, int32_t* __restrict__ part_c, float* __restrict__ aux,
              Control* ctl) {
  __shared__ float blk_p_w[8][256];
  __shared__ int32_t blk_c_w[8][256];
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
  const int t_begin = blockIdx.x * kRouteSelectTokensPerBlock;
  const int t_end = min(T, t_begin + kRouteSelectTokensPerBlock);
  for (int t = t_begin + warp; t < t_end; t += 8) {
    float v[EPL];
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
      const int e = lane + 32 * q;
      v[q] = e < E ? logits_in[static_cast<size_t>(t) * E + e] + bq[q] : -INFINITY;
      if (logits_out != nullptr && e < E) logits_out[static_cast<size_t>(t) * E + e] = v[q];
    }
    float m = -INFINITY;
#pragma unroll
    for (int q = 0; q < EPL; ++q) m = fmaxf(m, v[q]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
    float ex[EPL], s = 0.f;
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
      ex[q] = (lane + 32 * q < E) ? expf(v[q] - m) : 0.f;
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
        if (probs_out != nullptr) probs_out[static_cast<size_t>(t) * E + e] = p[q];
      }
    }
    unsigned taken = 0;
    float wsum = 0.f;
    int my_e = 0;
    float my_p = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < k) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
          const int e = lane + 32 * q;
          if (e < E && !((taken >> q) & 1u) && better(v[q], e, bv, be)) { bv = v[q]; be = e; }
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
          const float ov = __shfl_xor_sync(kFull, bv, off);
          const int oe = __shfl_xor_sync(kFull, be, off);
          if (better(ov, oe, bv, be)) { bv = ov; be = oe; }
        }
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
      idx_out[static_cast<size_t>(t) * k + lane] = my_e;
      w_out[static_cast<size_t>(t) * k + lane] = my_p / wsum;
    }
  }
#pragma unroll
  for (int q = 0; q < EPL; ++q) {
    const int e = lane + 32 * q;
    if (e < E) { blk_p_w[warp][e] = psum[q]; blk_c_w[warp][e] = cnt[q]; }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float a = 0.f;
    int c = 0;
    for (int w = 0; w < 8; ++w) { a += blk_p_w[w][e]; c += blk_c_w[w][e]; }
    tot_p[e] = a;
    tot_c[e] = c;
  }
  __syncthreads();
  block_partials_and_ticket(tot_p, tot_c, part_p, part_c, E, T, k, aux, ctl);
}

bool use_fused(int d, int E, moe_dtype_t dt) {
  (void)dt;
  const size_t bytes = static_cast<size_t>((d + 7) / 8) * 256;  // fp32 pairs, 256 B per 8 rows
  return E <= 8 && d % 8 == 0 && bytes <= 160 * 1024;
}

size_t fused_smem_bytes(int d) { return static_cast<size_t>((d + 7) / 8) * 256; }

}  // namespace

static int route_max_blocks(int T) {
  return std::max((T + kRouteSelectTokensPerBlock - 1) / kRouteSelectTokensPerBlock,
                  std::max(1, 2 * num_sms()));
}

size_t route_partials_bytes(int T, int E) {
  // Sized for the larger of the two paths' grids: sums then counts.
  return align_up(static_cast<size_t>(route_max_blocks(T)) * E * 4) * 2;
}

size_t route_logits_scratch_bytes(int T, int d, int E) {
  (void)d;
  return align_up(static_cast<size_t>(T) * E * 4);
}

cudaError_t launch_route(const void* x, const void* wg, const float* bias, moe_dtype_t dt, int T,
                         int d, int E, int k, int32_t* idx, float* w, float* aux, float* logits,
                         float* probs, float* logits_scratch, void* partials, Control* ctl,
                         cudaStream_t s) {
  const int nb_max = route_max_blocks(T);
  float* part_p = static_cast<float*>(partials);
  int32_t* part_c = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(partials) +
                                               align_up(static_cast<size_t>(nb_max) * E * 4));
  if (use_fused(d, E, dt)) {
    const int groups = (T + kFusedTokensPerGroup - 1) / kFusedTokensPerGroup;
    const int grid = std::max(1, std::min(groups, num_sms()));
    const size_t smem = fused_smem_bytes(d);
    if (dt == MOE_BF16) {
      auto kern = router_fused_e8<__nv_bfloat16>;
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      kern<<<grid, kFusedThreads, smem, s>>>(static_cast<const __nv_bfloat16*>(x),
                                             static_cast<const __nv_bfloat16*>(wg), bias, T, d, E, k,
                                             idx, w, logits, probs, part_p, part_c, aux, ctl);
    } else {
      auto kern = router_fused_e8<float>;
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      kern<<<grid, kFusedThreads, smem, s>>>(static_cast<const float*>(x), static_cast<const float*>(wg),
                                             bias, T, d, E, k, idx, w, logits, probs, part_p, part_c,
                                             aux, ctl);
    }
    return cudaGetLastError();
  }
  if (T > 0) {
    dim3 g1((T + 63) / 64, (E + 63) / 64);
    if (dt == MOE_BF16)
      router_gemm_tiled<__nv_bfloat16><<<g1, 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(wg), T, d, E,
          logits_scratch);
    else
      router_gemm_tiled<float><<<g1, 256, 0, s>>>(static_cast<const float*>(x),
                                                  static_cast<const float*>(wg), T, d, E,
                                                  logits_scratch);
  }
  const int g2 = std::max(1, (T + kRouteSelectTokensPerBlock - 1) / kRouteSelectTokensPerBlock);
  const int epl = (E + 31) / 32;
#define MOE_SELECT(N)                                                                        \
  router_select<N><<<g2, 256, 0, s>>>(logits_scratch, bias, T, E, k, idx, w, logits, probs, \
                                      part_p, part_c, aux, ctl)
  if (epl <= 1) MOE_SELECT(1);
  else if (epl <= 2) MOE_SELECT(2);
  else if (epl <= 4) MOE_SELECT(4);
  else MOE_SELECT(8);
#undef MOE_SELECT
  return cudaGetLastError();
}

}  // namespace moe
