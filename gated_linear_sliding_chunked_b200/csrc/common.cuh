// Shared device helpers for the hybrid attention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lz {

using bf16 = __nv_bfloat16;

// CTAs of `kern` resident on the device at once (SMs x blocks per SM), or 0
template <class Kern>
inline int resident_ctas(Kern kern, int threads, size_t smem) {
  int dev = 0, sms = 0, per = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kern, threads, smem) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return sms * per;
}

// Exponent span (in nats) of the cumulative log-gate inside one 16-row
// sub-block above which the factorized gate product q*exp(b_t-b_r) .
// k*exp(b_r-b_s) could leave the normal fp32/bf16 range; blocks beyond it
// take the elementwise exp(b_t - b_s) path.
constexpr float kSpanLimit = 60.0f;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

template <typename T>
__device__ __forceinline__ float ldf(const T* p) { return to_f(*p); }

// The gate as its logit (Gamma = sigma(z)): the log-gate is
// scale * log sigma(z), taken in the form that does not overflow for either
// sign of z, and dL/dz = dL/dg * scale * sigma(-z).
// (fast exp / log: when e^{-|z|} is below half an ulp of 1 the log term
// rounds to 0, an absolute error below 6e-8 in the log-gate)
__device__ __forceinline__ float gate_from_logit(float z, float scale) {
  return scale * (fminf(z, 0.f) - __logf(1.f + __expf(-fabsf(z))));
}
__device__ __forceinline__ float dlogit(float dg, float z, float scale) {
  return __fdividef(dg * scale, 1.f + __expf(z));
}
// Where a kernel reads the log-gates: fp32 log-gates, or bf16 logits mapped
// on the fly (passed by value to the strong-decay fallbacks, so that the
// log-gate instantiation keeps a one-pointer argument)
struct LogGates {
  const float* g;
  __device__ __forceinline__ float at(size_t i) const { return g[i]; }
};
struct LogitGates {
  const bf16* z;
  float s;
  __device__ __forceinline__ float at(size_t i) const { return gate_from_logit(__bfloat162float(z[i]), s); }
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

}  // namespace lz
