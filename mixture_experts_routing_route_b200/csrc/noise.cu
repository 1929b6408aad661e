// Random inputs of the router's training variants.
//
// Jitter: "MegaBlocks 01 - why MoE is hard", section 5 (during training the
// router input is multiplied by uniform noise in [1 - eps, 1 + eps]).
// Logit noise: "Integrating MoE into your model with Colossal-AI", step 2
// (NormalNoiseGenerator adds Gaussian noise to the router logits, scaled by
// the number of experts; the scale is the caller's std).
//
// Both draw from Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
// numbers: as easy as 1, 2, 3", SC 2011), a counter-based generator: the
// value of element n depends only on (n, seed), so any thread can produce any
// element and the stream does not depend on the launch shape.
//   jitter  element n = t*d + i: call n/4 on counter (lo, hi, 0, 0), word n%4;
//           u = (word >> 8) * 2^-24, m = (1 - eps) + (2 eps) * u (fp32, each
//           operation rounded), x' = x * m (fp32), rounded to bf16 for bf16.
//   noise   logit n = t*E + e: call n/2 on counter (lo, hi, 1, 0), words
//           2(n%2) and 2(n%2)+1; u1 = ((w0 >> 8) + 1) * 2^-24 in (0, 1],
//           u2 = (w1 >> 8) * 2^-24; z = sqrt(-2 ln u1) cos(2 pi u2) (Box and
//           Muller 1958); noise = std * z (fp32).
#include "common.cuh"

namespace moe {
namespace {

struct Philox4 {
  uint32_t v[4];
};

// Ten rounds: words 0 and 2 are multiplied by the two round constants; the
// high halves are mixed with words 1 and 3 and the key; the key advances by
// the two Weyl increments after every round.
__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                                 uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t lo0 = c0 * 0xD2511F53u, hi0 = __umulhi(c0, 0xD2511F53u);
    const uint32_t lo1 = c2 * 0xCD9E8D57u, hi1 = __umulhi(c2, 0xCD9E8D57u);
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  Philox4 out;
  out.v[0] = c0;
  out.v[1] = c1;
  out.v[2] = c2;
  out.v[3] = c3;
  return out;
}

template <typename T>
struct JitterIO;
template <> struct JitterIO<float> {
  static __device__ __forceinline__ float load(const float* p) { return __ldg(p); }
  static __device__ __forceinline__ void store(float* p, float v) { *p = v; }
};
template <> struct JitterIO<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};

// One thread per Philox call (4 elements).
template <typename T>
__global__ void __launch_bounds__(256)
jitter_kernel(const T* __restrict__ x, long long n, float eps, uint32_t k0, uint32_t k1,
              T* __restrict__ out) {
  pdl_begin();
  const float a = __fsub_rn(1.0f, eps), b = __fmul_rn(2.0f, eps);
  for (long long call = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
       call * 4 < n; call += static_cast<long long>(gridDim.x) * blockDim.x) {
    const Philox4 r = philox4x32_10(static_cast<uint32_t>(call), static_cast<uint32_t>(call >> 32),
                                    0u, 0u, k0, k1);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const long long i = call * 4 + j;
      if (i < n) {
        const float u = static_cast<float>(r.v[j] >> 8) * 5.9604644775390625e-8f;  // 2^-24
        const float m = __fadd_rn(a, __fmul_rn(b, u));
        JitterIO<T>::store(out + i, __fmul_rn(JitterIO<T>::load(x + i), m));
      }
    }
  }
}

// One thread per Philox call (2 logits).
__global__ void __launch_bounds__(256)
noise_kernel(long long n, float std, uint32_t k0, uint32_t k1, float* __restrict__ out) {
  pdl_begin();
  for (long long call = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
       call * 2 < n; call += static_cast<long long>(gridDim.x) * blockDim.x) {
    const Philox4 r = philox4x32_10(static_cast<uint32_t>(call), static_cast<uint32_t>(call >> 32),
                                    1u, 0u, k0, k1);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const long long i = call * 2 + j;
      if (i < n) {
        const float u1 = static_cast<float>((r.v[2 * j] >> 8) + 1u) * 5.9604644775390625e-8f;
        const float u2 = static_cast<float>(r.v[2 * j + 1] >> 8) * 5.9604644775390625e-8f;
        const float z = sqrtf(-2.0f * logf(u1)) * cosf(6.283185307179586f * u2);
        out[i] = std * z;
      }
    }
  }
}

int grid_for(long long calls) {
  const long long per = 256;
  const long long g = (calls + per - 1) / per;
  return static_cast<int>(g < 8LL * num_sms() ? (g < 1 ? 1 : g) : 8LL * num_sms());
}

}  // namespace

cudaError_t launch_jitter(const void* x, moe_dtype_t dt, long long n, float eps, uint64_t seed,
                          void* out, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  const int g = grid_for((n + 3) / 4);
  if (dt == MOE_BF16)
    return launch_pdl(jitter_kernel<__nv_bfloat16>, dim3(g), dim3(256), 0, s, false,
                      static_cast<const __nv_bfloat16*>(x), n, eps, k0, k1,
                      static_cast<__nv_bfloat16*>(out));
  return launch_pdl(jitter_kernel<float>, dim3(g), dim3(256), 0, s, false,
                    static_cast<const float*>(x), n, eps, k0, k1, static_cast<float*>(out));
}

cudaError_t launch_logit_noise(long long n, float std, uint64_t seed, float* out, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  return launch_pdl(noise_kernel, dim3(grid_for((n + 1) / 2)), dim3(256), 0, s, false, n, std, k0,
                    k1, out);
}

}  // namespace moe
