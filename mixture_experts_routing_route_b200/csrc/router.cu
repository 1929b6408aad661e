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

// Reduce the aux partials of all blocks (fixed block order, float64), then
// aux = E * sum_e f_e * P_e. Run by every thread of the last block.
__device__ void finalize_aux(const float* part_p, const int32_t* part_c, int nblk, int E, int T,
                             int k, float* aux) {
  __shared__ double red[256];
  double v = 0.0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    double ps = 0.0;
    long long cs = 0;
    for (int b = 0; b < nblk; ++b) {
      ps += static_cast<double>(__ldcg(part_p + static_cast<size_t>(b) * E + e));
      cs += __ldcg(part_c + static_cast<size_t>(b) * E + e);
    }
    const double P = T > 0 ? ps / T : 0.0;
    const double f = T > 0 ? static_cast<double>(cs) / (static_cast<double>(T) * k) : 0.0;
    v += f * P;
  }
  red[threadIdx.x] = v;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
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

// Shared-memory slot of Wg row i (8 experts, one 16-byte chunk per row for
// bf16): XOR-swizzled so the 8 lanes of a quarter-warp, which read rows
// 8l + j, hit 8 different bank groups.
__device__ __forceinline__ int wg_row_slot_bf16(int i) { return i ^ ((i >> 3) & 7); }

template <typename Tin>
__global__ void __launch_bounds__(256)
router_fused_e8(const Tin* __restrict__ x, const Tin* __restrict__ wg, const float* __restrict__ bias,
                int T, int d, int E, int k, int32_t* __restrict__ idx_out, float* __restrict__ w_out,
                float* __restrict__ logits_out, float* __restrict__ probs_out,
                float* __restrict__ part_p, int32_t* __restrict__ part_c, float* __restrict__ aux,
                Control* ctl) {
  constexpr int V = VecTraits<Tin>::kVec;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ float blk_p[8][8];
  __shared__ int32_t blk_c[8][8];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;

  // Stage Wg as [d][8] (zero for experts >= E).
  if constexpr (sizeof(Tin) == 2) {
    if (E == 8) {
      // one 16-byte row per load, rows in flight across the whole block
      const uint4* src = reinterpret_cast<const uint4*>(wg);
      uint4* dst = reinterpret_cast<uint4*>(smem_raw);
#pragma unroll 8
      for (int r = threadIdx.x; r < d; r += blockDim.x) dst[wg_row_slot_bf16(r)] = __ldg(src + r);
    } else {
      uint16_t* ws = reinterpret_cast<uint16_t*>(smem_raw);
      const uint16_t* wgu = reinterpret_cast<const uint16_t*>(wg);
      for (int i = threadIdx.x; i < d * 8; i += blockDim.x) {
        const int r = i >> 3, e = i & 7;
        ws[wg_row_slot_bf16(r) * 8 + e] = e < E ? wgu[static_cast<size_t>(r) * E + e] : uint16_t(0);
      }
    }
  } else {
    float* ws = reinterpret_cast<float*>(smem_raw);
    for (int i = threadIdx.x; i < d * 8; i += blockDim.x) {
      const int r = i >> 3, e = i & 7;
      ws[i] = e < E ? static_cast<float>(wg[static_cast<size_t>(r) * E + e]) : 0.f;
    }
  }
  __syncthreads();

  // lane -> (token-in-quad tq, expert e) after the reduce-scatter
  const int tq = lane >> 3;
  const int e = lane & 7;
  const bool e_ok = e < E;
  const float b_e = (bias != nullptr && e_ok) ? bias[e] : 0.f;
  float psum = 0.f;
  int cnt = 0;

  const int groups = (T + 31) / 32;
  for (int g = blockIdx.x; g < groups; g += gridDim.x) {
    const int t_base = g * 32 + warp * 4;
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.f;

    for (int i0 = lane * V; i0 < d; i0 += 32 * V) {
      float xv[4][V];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int t = t_base + q;
        uint4 u = make_uint4(0, 0, 0, 0);
        if (t < T) u = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d + i0));
        VecTraits<Tin>::unpack(u, xv[q]);
      }
#pragma unroll
      for (int j = 0; j < V; ++j) {
        float wr[8];
        if constexpr (sizeof(Tin) == 2) {
          const uint4 u = reinterpret_cast<const uint4*>(smem_raw)[wg_row_slot_bf16(i0 + j)];
          VecTraits<__nv_bfloat16>::unpack(u, wr);
        } else {
          const float4* p = reinterpret_cast<const float4*>(smem_raw) + (i0 + j) * 2;
          const float4 a = p[0], b = p[1];
          wr[0] = a.x; wr[1] = a.y; wr[2] = a.z; wr[3] = a.w;
          wr[4] = b.x; wr[5] = b.y; wr[6] = b.z; wr[7] = b.w;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int ee = 0; ee < 8; ++ee) acc[q * 8 + ee] = fmaf(xv[q][j], wr[ee], acc[q * 8 + ee]);
      }
    }
    // Reduce-scatter over the warp: afterwards lane l holds the full sum of acc[l].
#pragma unroll
    for (int half = 16; half >= 1; half >>= 1) {
      const bool upper = (lane & half) != 0;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float send = upper ? acc[i] : acc[i + half];
        const float keep = upper ? acc[i + half] : acc[i];
        acc[i] = keep + __shfl_xor_sync(kFull, send, half);
      }
    }
    const int t = t_base + tq;
    const bool t_ok = t < T;
    float v = e_ok ? acc[0] + b_e : -INFINITY;
    if (logits_out != nullptr && t_ok && e_ok) logits_out[static_cast<size_t>(t) * E + e] = v;

    // softmax inside the 8-lane group of token t
    float m = v;
#pragma unroll
    for (int off = 4; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
    const float ex = e_ok ? expf(v - m) : 0.f;
    float s = ex;
#pragma unroll
    for (int off = 4; off >= 1; off >>= 1) s += __shfl_xor_sync(kFull, s, off);
    const float p = ex / s;
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
  // Warp totals per expert: lanes e, e+8, e+16, e+24 hold the same expert.
  psum += __shfl_xor_sync(kFull, psum, 8);
  psum += __shfl_xor_sync(kFull, psum, 16);
  cnt += __shfl_xor_sync(kFull, cnt, 8);
  cnt += __shfl_xor_sync(kFull, cnt, 16);
  if (lane < 8) {
    blk_p[warp][lane] = psum;
    blk_c[warp][lane] = cnt;
  }
  __syncthreads();
  __shared__ float tot_p[8];
  __shared__ int32_t tot_c[8];
  if (threadIdx.x < 8) {
    float a = 0.f;
    int c = 0;
    for (int w = 0; w < 8; ++w) { a += blk_p[w][threadIdx.x]; c += blk_c[w][threadIdx.x]; }
    tot_p[threadIdx.x] = a;
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
  const size_t bytes = static_cast<size_t>(d) * 8 * (dt == MOE_BF16 ? 2 : 4);
  return E <= 8 && bytes <= 96 * 1024;
}

}  // namespace

int route_num_blocks(int T, int E) {
  // Fused path: a persistent grid of at most two blocks per SM.
  const int groups = (T + 31) / 32;
  if (E <= 8) return std::max(1, std::min(groups, 2 * num_sms()));
  return std::max(1, (T + kRouteSelectTokensPerBlock - 1) / kRouteSelectTokensPerBlock);
}

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
    const int groups = (T + 31) / 32;
    const int grid = std::max(1, std::min(groups, 2 * num_sms()));
    const size_t smem = static_cast<size_t>(d) * 8 * (dt == MOE_BF16 ? 2 : 4);
    if (dt == MOE_BF16) {
      auto kern = router_fused_e8<__nv_bfloat16>;
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      kern<<<grid, 256, smem, s>>>(static_cast<const __nv_bfloat16*>(x),
                                   static_cast<const __nv_bfloat16*>(wg), bias, T, d, E, k, idx, w,
                                   logits, probs, part_p, part_c, aux, ctl);
    } else {
      auto kern = router_fused_e8<float>;
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      kern<<<grid, 256, smem, s>>>(static_cast<const float*>(x), static_cast<const float*>(wg), bias,
                                   T, d, E, k, idx, w, logits, probs, part_p, part_c, aux, ctl);
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
