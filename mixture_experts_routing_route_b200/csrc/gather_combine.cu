// Gather (x rows into expert-contiguous order) and the weighted combine.
//
// Gather: "MegaBlocks 01", section 4.3 (binned_gather reorders [tokens, hs]
// by the sort; the token of flat slot s is s / top_k), here without padding.
// A warp per row, 16-byte vectors through registers (see gather_lsu).
//
// Combine: "ops-transformer MoE operators", 原理 Step 4 (weighted sum of the
// chosen experts' outputs) and "MegaBlocks 01", sections 4.3 and 5 (multiply by
// the router weight and sum over top-k; dropped slots contribute zero). The
// kernel gathers each token's k rows instead of scattering: every output
// element is written once, by one thread, in a fixed j order (no atomics).
#include "common.cuh"
#include <algorithm>

namespace moe {

namespace {

// Gather kernel: a warp per row (the gathered rows first, then, when the
// combine runs in the down projection, the output rows to zero), 16-byte
// loads and stores through registers, each lane holding up to 16 vectors of
// an 8 KB chunk in flight, 8 warps per block and up to 8 blocks per SM. A
// padding row of the binned layout (row_slot -1) is written as zeros, and so
// is the layer output row of a token whose every slot was dropped; any other
// bad slot index is reported and its row skipped. (A version driving bulk
// copies through a shared-memory ring from one lane per warp measured the
// same at 8 KB rows and 2.5x slower at 2 KB rows, with 4 copies in flight
// per SM.)
constexpr int kGatherLsuWarps = 8;
constexpr int kGatherLsuVec = 16;  // vectors per lane per chunk

__global__ void __launch_bounds__(kGatherLsuWarps * 32)
gather_lsu(const uint8_t* __restrict__ x, uint32_t row_bytes, int T, int k,
           const int32_t* __restrict__ row_slot, const int32_t* __restrict__ seg, int E,
           long long rows_max, int binned, uint8_t* __restrict__ x_perm,
           const int32_t* __restrict__ slot_to_row, uint8_t* __restrict__ zero_out, Control* ctl) {
  pdl_begin();
  const int lane = threadIdx.x & 31;
  long long R = __ldg(seg + E);
  if (R > rows_max || R < 0) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_error(ctl, MOE_DEVERR_ROW_RANGE);
    R = R < 0 ? 0 : rows_max;
  }
  if (x_perm == nullptr) R = 0;  // the up projection gathers: output zeroing only
  const long long S = static_cast<long long>(T) * k;
  const long long total = R + (zero_out != nullptr ? static_cast<long long>(T) : 0);
  const uint32_t nvec = row_bytes / 16;
  const long long gw = static_cast<long long>(blockIdx.x) * kGatherLsuWarps + (threadIdx.x >> 5);
  const long long tw = static_cast<long long>(gridDim.x) * kGatherLsuWarps;
  for (long long u = gw; u < total; u += tw) {
    const uint4* src = nullptr;
    uint4* dst;
    if (u >= R) {  // output row of token t: zero when none of its k slots was kept
      const long long t = u - R;
      bool kept = false;
      for (int j = 0; j < k; ++j) kept |= __ldg(slot_to_row + t * k + j) >= 0;
      if (kept) continue;
      dst = reinterpret_cast<uint4*>(zero_out + static_cast<size_t>(t) * row_bytes);
    } else {
      const int slot = __ldg(row_slot + u);
      dst = reinterpret_cast<uint4*>(x_perm + static_cast<size_t>(u) * row_bytes);
      if (!(binned && slot == -1)) {
        if (slot < 0 || slot >= S) {
          if (lane == 0) set_error(ctl, MOE_DEVERR_ROW_RANGE);
          continue;
        }
        src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(slot / k) * row_bytes);
      }
    }
    for (uint32_t base = 0; base < nvec; base += 32 * kGatherLsuVec) {
      uint4 v[kGatherLsuVec];
#pragma unroll
      for (int i = 0; i < kGatherLsuVec; ++i) {
        const uint32_t j = base + i * 32 + lane;
        v[i] = (src != nullptr && j < nvec) ? __ldg(src + j) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int i = 0; i < kGatherLsuVec; ++i) {
        const uint32_t j = base + i * 32 + lane;
        if (j < nvec) dst[j] = v[i];
      }
    }
  }
}

template <typename T>
struct CombineVec;
template <> struct CombineVec<__nv_bfloat16> {
  static constexpr int kVec = 8;
  static __device__ __forceinline__ void fma(const uint4& u, float w, float (&a)[8]) {
    const uint32_t v[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a[2 * i] = fmaf(w, __uint_as_float(v[i] << 16), a[2 * i]);
      a[2 * i + 1] = fmaf(w, __uint_as_float(v[i] & 0xffff0000u), a[2 * i + 1]);
    }
  }
  static __device__ __forceinline__ uint4 pack(const float (&a)[8]) {
    uint32_t v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(a[2 * i], a[2 * i + 1]);
      v[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    return make_uint4(v[0], v[1], v[2], v[3]);
  }
};
template <> struct CombineVec<float> {
  static constexpr int kVec = 4;
  static __device__ __forceinline__ void fma(const uint4& u, float w, float (&a)[4]) {
    a[0] = fmaf(w, __uint_as_float(u.x), a[0]);
    a[1] = fmaf(w, __uint_as_float(u.y), a[1]);
    a[2] = fmaf(w, __uint_as_float(u.z), a[2]);
    a[3] = fmaf(w, __uint_as_float(u.w), a[3]);
  }
  static __device__ __forceinline__ uint4 pack(const float (&a)[4]) {
    return make_uint4(__float_as_uint(a[0]), __float_as_uint(a[1]), __float_as_uint(a[2]),
                      __float_as_uint(a[3]));
  }
};

constexpr int kCombineThreads = 128;

// Each thread owns up to two 16-byte column vectors of one token and requests
// the K rows of both before it accumulates. A token needs tpt threads (its
// d/V vectors, two per thread). When tpt <= the block, a block takes
// 128/tpt whole tokens (grid.x = token groups); otherwise one token spreads
// over grid.y blocks. K is the compile-time top-k (0: runtime k, rows one by
// one).
template <typename T, int K>
__global__ void __launch_bounds__(kCombineThreads)
combine_gather(const T* __restrict__ y, const float* __restrict__ w,
               const int32_t* __restrict__ slot_to_row, int T_, int d, int k_rt, int tpt,
               long long rows_max, T* __restrict__ out, Control* ctl) {
  pdl_begin();
  constexpr int V = CombineVec<T>::kVec;
  constexpr int NV = 2;  // column vectors per thread
  const int k = K > 0 ? K : k_rt;
  int t, v0, vstride;
  if (tpt <= kCombineThreads) {
    const int tpb = kCombineThreads / tpt;
    const int local = threadIdx.x / tpt;
    if (local >= tpb) return;
    t = blockIdx.x * tpb + local;
    v0 = threadIdx.x - local * tpt;
    vstride = tpt;
  } else {
    t = blockIdx.x;
    v0 = blockIdx.y * kCombineThreads * NV + threadIdx.x;
    vstride = kCombineThreads;
  }
  const int col0 = v0 * V;
  if (t >= T_ || col0 >= d) return;
  int rows[K > 0 ? K : 1];
  float wj[K > 0 ? K : 1];
  float acc[NV][V];
#pragma unroll
  for (int c = 0; c < NV; ++c)
#pragma unroll
    for (int i = 0; i < V; ++i) acc[c][i] = 0.f;
  if constexpr (K > 0) {
#pragma unroll
    for (int j = 0; j < K; ++j) {
      rows[j] = __ldg(slot_to_row + static_cast<size_t>(t) * K + j);
      wj[j] = __ldg(w + static_cast<size_t>(t) * K + j);
      if (rows[j] >= rows_max) {
        if (col0 == 0) set_error(ctl, MOE_DEVERR_ROW_RANGE);
        rows[j] = -1;
      }
    }
    uint4 u[K][NV];
#pragma unroll
    for (int j = 0; j < K; ++j)
#pragma unroll
      for (int c = 0; c < NV; ++c) {
        const int col = (v0 + c * vstride) * V;
        u[j][c] = make_uint4(0, 0, 0, 0);
        if (rows[j] >= 0 && col < d)
          u[j][c] = __ldg(reinterpret_cast<const uint4*>(y + static_cast<size_t>(rows[j]) * d + col));
      }
#pragma unroll
    for (int j = 0; j < K; ++j)
      if (rows[j] >= 0)
#pragma unroll
        for (int c = 0; c < NV; ++c) CombineVec<T>::fma(u[j][c], wj[j], acc[c]);
  } else {
    for (int j = 0; j < k; ++j) {
      const int row = __ldg(slot_to_row + static_cast<size_t>(t) * k + j);
      if (row < 0) continue;
      if (row >= rows_max) {
        if (col0 == 0) set_error(ctl, MOE_DEVERR_ROW_RANGE);
        continue;
      }
      const float wv = __ldg(w + static_cast<size_t>(t) * k + j);
#pragma unroll
      for (int c = 0; c < NV; ++c) {
        const int col = (v0 + c * vstride) * V;
        if (col < d)
          CombineVec<T>::fma(__ldg(reinterpret_cast<const uint4*>(y + static_cast<size_t>(row) * d + col)),
                             wv, acc[c]);
      }
    }
  }
#pragma unroll
  for (int c = 0; c < NV; ++c) {
    const int col = (v0 + c * vstride) * V;
    if (col < d)
      *reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * d + col) = CombineVec<T>::pack(acc[c]);
  }
}

template <typename T>
cudaError_t launch_combine_t(const T* y, const float* w, const int32_t* s2r, int T_, int d, int k,
                      long long rows_max, T* out, Control* ctl, cudaStream_t s) {
  constexpr int V = CombineVec<T>::kVec;
  const int nvec = (d + V - 1) / V;
  const int tpt = (nvec + 1) / 2;  // threads per token, two vectors each
  const dim3 grid = tpt <= kCombineThreads
                        ? dim3((T_ + kCombineThreads / tpt - 1) / (kCombineThreads / tpt), 1)
                        : dim3(T_, (d + kCombineThreads * V * 2 - 1) / (kCombineThreads * V * 2));
  auto kern = combine_gather<T, 0>;
  switch (k) {
    case 1: kern = combine_gather<T, 1>; break;
    case 2: kern = combine_gather<T, 2>; break;
    case 4: kern = combine_gather<T, 4>; break;
    case 8: kern = combine_gather<T, 8>; break;
    default: break;
  }
  return launch_pdl(kern, grid, dim3(kCombineThreads), 0, s, false, y, w, s2r, T_, d, k, tpt,
                    rows_max, out, ctl);
}

}  // namespace

cudaError_t launch_gather(const void* x, size_t elem, int T, int d, int k, const int32_t* row_slot,
                          const int32_t* seg, int E, int64_t rows_max, void* x_perm, Control* ctl,
                          cudaStream_t s, bool binned, const int32_t* slot_to_row, void* zero_out) {
  if (T <= 0 || (rows_max <= 0 && zero_out == nullptr)) return cudaSuccess;
  const uint32_t row_bytes = static_cast<uint32_t>(static_cast<size_t>(d) * elem);
  const long long units = (x_perm != nullptr ? rows_max : 0) + (zero_out != nullptr ? T : 0);
  const int g = static_cast<int>(std::max<long long>(
      1, std::min<long long>((units + kGatherLsuWarps - 1) / kGatherLsuWarps, 8LL * num_sms())));
  return launch_pdl(gather_lsu, dim3(g), dim3(kGatherLsuWarps * 32), 0, s, false,
                    static_cast<const uint8_t*>(x), row_bytes, T, k, row_slot, seg, E, rows_max,
                    binned ? 1 : 0, static_cast<uint8_t*>(x_perm), slot_to_row,
                    static_cast<uint8_t*>(zero_out), ctl);
}

cudaError_t launch_combine(const void* y, const float* w, const int32_t* slot_to_row, size_t elem,
                           int T, int d, int k, int64_t rows_max, void* out, Control* ctl,
                           cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if (elem == 2)
    return launch_combine_t<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(y), w, slot_to_row, T,
                                           d, k, rows_max, static_cast<__nv_bfloat16*>(out), ctl, s);
  return launch_combine_t<float>(static_cast<const float*>(y), w, slot_to_row, T, d, k, rows_max,
                                 static_cast<float*>(out), ctl, s);
}

}  // namespace moe
