// Stage-1 distillation loss: the mean squared error between the hybrid
// attention output and the teacher's attention output ("Lizard: An Efficient
// Linearization Framework for Large Language Models", technical summary
// section 2b, training strategy, first stage), with its gradient
// dO = 2 (o - target) / n for the backward.
//
// The bf16 tensor-core forward computes the per-chunk sums inside the output
// kernel's epilogue; every other path runs launch_mse_generic over the stored
// output.  Both end in launch_loss_reduce, which adds the partial sums in a
// fixed order in fp64, so the loss is reproducible bit for bit.
#include "common.cuh"
#include "kernels.h"

namespace lz {
namespace {

constexpr int kMseThreads = 256;
constexpr int kReduceThreads = 256;

template <typename IO>
__global__ void __launch_bounds__(kMseThreads) mse_generic_kernel(const IO* o, const IO* target, IO* dO,
                                                                   float scale, size_t n, float* part) {
  __shared__ float wsum[kMseThreads / 32];
  float acc = 0.f;
  const size_t stride = (size_t)gridDim.x * kMseThreads;
  for (size_t x = (size_t)blockIdx.x * kMseThreads + threadIdx.x; x < n; x += stride) {
    const float e = to_f(o[x]) - to_f(target[x]);
    acc = fmaf(e, e, acc);
    if (dO) dO[x] = from_f<IO>(scale * e);
  }
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kMseThreads / 32; ++w) tot += wsum[w];
    part[blockIdx.x] = tot;
  }
}

__global__ void __launch_bounds__(kReduceThreads) loss_reduce_kernel(const float* part, size_t nparts,
                                                                     double inv_n, float* loss) {
  __shared__ double red[kReduceThreads];
  double acc = 0.0;
  for (size_t x = threadIdx.x; x < nparts; x += kReduceThreads) acc += (double)part[x];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int h = kReduceThreads / 2; h > 0; h >>= 1) {
    if ((int)threadIdx.x < h) red[threadIdx.x] += red[threadIdx.x + h];
    __syncthreads();
  }
  if (threadIdx.x == 0) loss[0] = (float)(red[0] * inv_n);
}

}  // namespace

int mse_generic_parts(size_t n) {
  const size_t blocks = (n + kMseThreads - 1) / kMseThreads;
  return (int)(blocks < (size_t)kMseParts ? blocks : (size_t)kMseParts);
}

cudaError_t launch_mse_generic(const void* o, const void* target, void* dO, float scale, size_t n,
                               bool is_bf16, float* part, cudaStream_t s) {
  const int blocks = mse_generic_parts(n);
  if (blocks == 0) return cudaSuccess;
  ScopedTiming tm("mse_loss", s);
  if (is_bf16)
    mse_generic_kernel<bf16><<<blocks, kMseThreads, 0, s>>>((const bf16*)o, (const bf16*)target, (bf16*)dO,
                                                            scale, n, part);
  else
    mse_generic_kernel<float><<<blocks, kMseThreads, 0, s>>>((const float*)o, (const float*)target,
                                                             (float*)dO, scale, n, part);
  return cudaGetLastError();
}

cudaError_t launch_loss_reduce(const float* part, size_t nparts, double inv_n, float* loss,
                               cudaStream_t s) {
  ScopedTiming tm("loss_reduce", s);
  loss_reduce_kernel<<<1, kReduceThreads, 0, s>>>(part, nparts, inv_n, loss);
  return cudaGetLastError();
}

}  // namespace lz
