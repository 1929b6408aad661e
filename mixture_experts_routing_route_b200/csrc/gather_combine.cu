// Gather (x rows into expert-contiguous order) and the weighted combine.
//
// Gather: "MegaBlocks 01", section 4.3 (binned_gather reorders [tokens, hs]
// by the sort; the token of flat slot s is s / top_k), here without padding.
// Each warp's lane 0 drives a ring of 6 shared-memory buffers with bulk (TMA)
// copies: cp.async.bulk global->shared completing on an mbarrier, then
// cp.async.bulk shared->global into the gathered row. A buffer is refilled one
// iteration after its store was issued, so loads and a store are always in
// flight together. No multicast.
//
// Combine: "ops-transformer MoE operators", 原理 Step 4 (weighted sum of the
// chosen experts' outputs) and "MegaBlocks 01", sections 4.3 and 5 (multiply by
// the router weight and sum over top-k; dropped slots contribute zero). The
// kernel gathers each token's k rows instead of scattering: every output
// element is written once, by one thread, in a fixed j order (no atomics).
#include "common.cuh"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kGatherWarps = 4;
constexpr int kGatherBufs = 6;
constexpr int kGatherPiece = 8192;  // bytes per buffer

__global__ void __launch_bounds__(kGatherWarps * 32)
gather_bulk(const uint8_t* __restrict__ x, uint32_t row_bytes, int T, int k,
            const int32_t* __restrict__ row_slot, const int32_t* __restrict__ seg, int E,
            long long rows_max, int binned, uint8_t* __restrict__ x_perm,
            const int32_t* __restrict__ slot_to_row, uint8_t* __restrict__ zero_out, Control* ctl) {
  pdl_begin();
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t bars[kGatherWarps][kGatherBufs];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // Binned layout: a padding row (row_slot -1) is stored from a zero piece;
  // so is the layer output row of a token whose every slot was dropped, when
  // the combine runs in the down projection (zero_out = the output).
  uint8_t* zero = smem + static_cast<size_t>(kGatherWarps) * kGatherBufs * kGatherPiece;
  if (binned || zero_out != nullptr) {
    for (int i = threadIdx.x; i < kGatherPiece / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(zero)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();  // generic writes, read by the bulk stores
  }
  __syncthreads();
  if (lane != 0) return;

  long long R = __ldg(seg + E);
  if (R > rows_max || R < 0) {
    set_error(ctl, MOE_DEVERR_ROW_RANGE);
    R = R < 0 ? 0 : rows_max;
  }
  if (x_perm == nullptr) R = 0;  // the up projection gathers: output zeroing only
  const long long S = static_cast<long long>(T) * k;
  const uint32_t ppr = (row_bytes + kGatherPiece - 1) / kGatherPiece;  // pieces per row
  const long long rowp = R * ppr;  // pieces of gathered rows, then of output rows
  const long long total = rowp + (zero_out != nullptr ? static_cast<long long>(T) * ppr : 0);
  const long long gw = static_cast<long long>(blockIdx.x) * kGatherWarps + warp;
  const long long tw = static_cast<long long>(gridDim.x) * kGatherWarps;
  if (gw >= total) return;
  const long long mine = (total - gw + tw - 1) / tw;

  uint8_t* buf0 = smem + static_cast<size_t>(warp) * kGatherBufs * kGatherPiece;
  for (int b = 0; b < kGatherBufs; ++b) mbar_init(&bars[warp][b], 1);
  fence_mbar_init();

  // Source / destination / size of the i-th piece of this warp. A padding
  // row of the binned layout has no source (src null: stored from zero); any
  // other bad slot index is reported and the piece is skipped (size 0).
  auto piece = [&](long long i, const uint8_t*& src, uint8_t*& dst, uint32_t& bytes) {
    const long long p = gw + i * tw;
    if (p >= rowp) {  // output row of token t: zero when none of its k slots was kept
      const long long q = p - rowp, t = q / ppr;
      const uint32_t off = static_cast<uint32_t>(q % ppr) * kGatherPiece;
      bool kept = false;
      for (int j = 0; j < k; ++j) kept |= __ldg(slot_to_row + t * k + j) >= 0;
      bytes = kept ? 0u : min(static_cast<uint32_t>(kGatherPiece), row_bytes - off);
      src = nullptr;
      dst = zero_out + static_cast<size_t>(t) * row_bytes + off;
      return;
    }
    const long long row = p / ppr;
    const uint32_t off = static_cast<uint32_t>(p % ppr) * kGatherPiece;
    const int slot = __ldg(row_slot + row);
    bytes = min(static_cast<uint32_t>(kGatherPiece), row_bytes - off);
    if (binned && slot == -1) {
      src = nullptr;
      dst = x_perm + static_cast<size_t>(row) * row_bytes + off;
      return;
    }
    if (slot < 0 || slot >= S) {
      set_error(ctl, MOE_DEVERR_ROW_RANGE);
      bytes = 0;
      return;
    }
    src = x + static_cast<size_t>(slot / k) * row_bytes + off;
    dst = x_perm + static_cast<size_t>(row) * row_bytes + off;
  };

  const uint8_t* srcs[kGatherBufs];
  uint8_t* dsts[kGatherBufs];
  uint32_t sizes[kGatherBufs];
  uint32_t phase = 0;     // bit b: parity to wait for on buffer b
  uint32_t inflight = 0;  // bit b: buffer b has a load not yet waited for
  const long long pro = mine < kGatherBufs ? mine : kGatherBufs;
  for (long long i = 0; i < pro; ++i) {
    piece(i, srcs[i], dsts[i], sizes[i]);
    if (sizes[i] && srcs[i]) {
      mbar_arrive_expect_tx(&bars[warp][i], sizes[i]);
      bulk_load(buf0 + i * kGatherPiece, srcs[i], sizes[i], &bars[warp][i]);
      inflight |= 1u << i;
    }
  }
  bool ok = true;
  for (long long i = 0; i < mine && ok; ++i) {
    const int b = static_cast<int>(i % kGatherBufs);
    bool committed = sizes[b] != 0;  // this iteration issues a store group
    if (sizes[b] && srcs[b] == nullptr) {
      bulk_store(dsts[b], zero, sizes[b]);
      bulk_commit();
    } else if (sizes[b]) {
      if (!mbar_wait_bounded(&bars[warp][b], (phase >> b) & 1u)) {
        set_error(ctl, MOE_DEVERR_TIMEOUT);
        ok = false;
        break;
      }
      phase ^= 1u << b;
      inflight &= ~(1u << b);
      bulk_store(dsts[b], buf0 + b * kGatherPiece, sizes[b]);
      bulk_commit();
    }
    // Refill the buffer of the previous piece (its store is one group older
    // than the one just issued), so a store and the loads overlap.
    const long long nxt = i - 1 + kGatherBufs;
    if (i >= 1 && nxt < mine) {
      const int pb = static_cast<int>((i - 1) % kGatherBufs);
      // the previous piece's store group must have read its buffer: when this
      // iteration issued a group, that is every group but the newest
      if (committed) bulk_wait_read<1>();
      else bulk_wait_read<0>();
      piece(nxt, srcs[pb], dsts[pb], sizes[pb]);
      if (sizes[pb] && srcs[pb]) {
        mbar_arrive_expect_tx(&bars[warp][pb], sizes[pb]);
        bulk_load(buf0 + pb * kGatherPiece, srcs[pb], sizes[pb], &bars[warp][pb]);
        inflight |= 1u << pb;
      }
    }
  }
  if (!ok) {
    // Let every load still in flight land (bounded) before the buffers go away.
    for (int b = 0; b < kGatherBufs; ++b)
      if ((inflight >> b) & 1u) (void)mbar_wait_bounded(&bars[warp][b], (phase >> b) & 1u);
  }
  bulk_wait<0>();
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
  // the ring of every warp, then one zero piece (binned padding rows)
  const size_t smem = static_cast<size_t>(kGatherWarps) * kGatherBufs * kGatherPiece + kGatherPiece;
  cudaFuncSetAttribute(gather_bulk, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  return launch_pdl(gather_bulk, dim3(num_sms()), dim3(kGatherWarps * 32), smem, s, false,
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
