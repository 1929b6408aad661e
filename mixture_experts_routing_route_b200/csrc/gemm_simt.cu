// Grouped expert GEMM for fp32 layers, on CUDA cores.
//
// The tensor cores have no fp32-input mode (tf32 keeps 10 mantissa bits), so
// an fp32 layer keeps full fp32 products on FFMA. Same segment/tile scheme as
// the tensor-core kernel: expert-contiguous rows, a device-side tile prefix,
// experts with no rows skipped. 64x64 output tiles, 256 threads of 4x4.
// "MegaBlocks 01", section 4.3 (bmm -> activation -> bmm per expert).
#include "common.cuh"
#include <cmath>

namespace moe {

namespace {

constexpr int TM = 64, TN = 64, TK = 16;
constexpr int kMaxE = 256;

enum { EPI_SWIGLU = 0, EPI_GELU = 1, EPI_STORE = 2 };

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + expf(-g)); }
__device__ __forceinline__ float gelu_f(float z) {
  return 0.5f * z * (1.0f + erff(z * 0.70710678118654752440f));
}

// grid.x = n tiles, grid.y = upper bound on m tiles (ceil(rows_max/64) + E).
template <int EPI>
__global__ void __launch_bounds__(256)
grouped_gemm_f32(const float* __restrict__ A, const float* __restrict__ B0,
                 const float* __restrict__ B1, const int32_t* __restrict__ seg, int E, int K, int N,
                 long long rows_max, float* __restrict__ Cout, Control* ctl) {
  pdl_begin();
  __shared__ int mt_start[kMaxE + 1];
  __shared__ int seg_s[kMaxE + 1];
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs0[TK][TN + 4];
  __shared__ float Bs1[TK][TN + 4];
  for (int i = threadIdx.x; i <= E; i += blockDim.x) seg_s[i] = __ldg(seg + i);
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      mt_start[e] = run;
      int m = seg_s[e + 1] - seg_s[e];
      if (m < 0 || seg_s[e] < 0 || seg_s[e + 1] > rows_max) {
        set_error(ctl, MOE_DEVERR_ROW_RANGE);
        m = 0;
      }
      run += (m + TM - 1) / TM;
    }
    mt_start[E] = run;
  }
  __syncthreads();
  const int mtile = blockIdx.y;
  if (mtile >= mt_start[E]) return;
  int e = 0;
  while (e + 1 < E && mt_start[e + 1] <= mtile) ++e;
  const int row0 = seg_s[e] + (mtile - mt_start[e]) * TM;
  const int rows = min(TM, seg_s[e + 1] - row0);
  const int n0 = blockIdx.x * TN;
  const float* Be0 = B0 + static_cast<size_t>(e) * K * N;
  const float* Be1 = EPI == EPI_SWIGLU ? B1 + static_cast<size_t>(e) * K * N : nullptr;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc0[4][4] = {}, acc1[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += TK) {
    for (int i = threadIdx.x; i < TM * TK; i += 256) {
      const int r = i / TK, kk = i % TK;
      As[kk][r] = (r < rows && k0 + kk < K) ? A[static_cast<size_t>(row0 + r) * K + k0 + kk] : 0.f;
    }
    for (int i = threadIdx.x; i < TK * TN; i += 256) {
      const int kk = i / TN, c = i % TN;
      const bool ok = k0 + kk < K && n0 + c < N;
      Bs0[kk][c] = ok ? Be0[static_cast<size_t>(k0 + kk) * N + n0 + c] : 0.f;
      if (EPI == EPI_SWIGLU) Bs1[kk][c] = ok ? Be1[static_cast<size_t>(k0 + kk) * N + n0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b0[4], b1[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        b0[i] = Bs0[kk][tx * 4 + i];
        if (EPI == EPI_SWIGLU) b1[i] = Bs1[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc0[i][j] = fmaf(a[i], b0[j], acc0[i][j]);
          if (EPI == EPI_SWIGLU) acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i;
    if (r >= rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = n0 + tx * 4 + j;
      if (c >= N) continue;
      float v = acc0[i][j];
      if (EPI == EPI_SWIGLU) v = silu_f(v) * acc1[i][j];
      else if (EPI == EPI_GELU) v = gelu_f(v);
      Cout[static_cast<size_t>(row0 + r) * N + c] = v;
    }
  }
}

template <int EPI>
cudaError_t run_f32(const float* A, const float* B0, const float* B1, int64_t rows_max, int K, int N,
             int E, const int32_t* seg, float* C, Control* ctl, cudaStream_t s) {
  const long long mt_bound = (rows_max + TM - 1) / TM + E;
  dim3 grid((N + TN - 1) / TN, static_cast<unsigned>(mt_bound));
  return launch_pdl(grouped_gemm_f32<EPI>, grid, dim3(256), 0, s, false, A, B0, B1, seg, E, K, N,
                    rows_max, C, ctl);
}

}  // namespace

cudaError_t launch_ffn_f32(const float* x_perm, const float* w1, const float* w3, const float* w2,
                           moe_act_t act, int64_t rows_max, int d, int F, int E,
                           const int32_t* seg, float* h, float* y, Control* ctl, cudaStream_t s,
                           cudaEvent_t after_up) {
  cudaError_t e = cudaSuccess;
  if (rows_max > 0) {
    if (act == MOE_ACT_SWIGLU)
      e = run_f32<EPI_SWIGLU>(x_perm, w1, w3, rows_max, d, F, E, seg, h, ctl, s);
    else
      e = run_f32<EPI_GELU>(x_perm, w1, nullptr, rows_max, d, F, E, seg, h, ctl, s);
  }
  if (e != cudaSuccess) return e;
  if (after_up) cudaEventRecord(after_up, s);
  if (rows_max > 0) e = run_f32<EPI_STORE>(h, w2, nullptr, rows_max, F, d, E, seg, y, ctl, s);
  return e;
}

}  // namespace moe
