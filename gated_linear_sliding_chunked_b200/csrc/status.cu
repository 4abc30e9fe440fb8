// The library's device status word: kernels whose waits are bounded (the
// tcgen05 kernels wait on mbarriers for their tensor-core work) add one to
// it for every wait that gave up instead of spinning on; lz_device_check
// reads and clears it.  One word per device, looked up once per device with
// cudaGetSymbolAddress (the symbol's host-side name is not a device address).
#include <cstdio>
#include <mutex>
#include <unordered_map>

#include "../../include/lizard.h"
#include "kernels.h"
#include "mma.cuh"
#include "tc05.cuh"

namespace {

static __device__ unsigned int g_status_word;

std::mutex g_mu;
std::unordered_map<int, unsigned int*> g_addr;  // device ordinal -> address of the word

}  // namespace

namespace lz {

unsigned int* device_status_word() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  auto it = g_addr.find(dev);
  if (it != g_addr.end()) return it->second;
  void* a = nullptr;
  if (cudaGetSymbolAddress(&a, g_status_word) != cudaSuccess || a == nullptr) return nullptr;
  g_addr.emplace(dev, static_cast<unsigned int*>(a));
  return static_cast<unsigned int*>(a);
}

}  // namespace lz

extern "C" lz_status lz_device_check(lz_stream stream) {
  unsigned int* word = lz::device_status_word();
  if (word == nullptr)
    return (lz_status)lz::set_last_error(LZ_ERR_CUDA, "lz_device_check: no device status word");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int n = 0;
  cudaError_t e = cudaMemcpyAsync(&n, word, sizeof(n), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && n != 0) e = cudaMemsetAsync(word, 0, sizeof(n), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    char msg[256];
    std::snprintf(msg, sizeof(msg), "lz_device_check: %s", cudaGetErrorString(e));
    return (lz_status)lz::set_last_error(LZ_ERR_CUDA, msg);
  }
  if (n != 0) {
    char msg[256];
    std::snprintf(msg, sizeof(msg), "lz_device_check: %u bounded device wait(s) gave up", n);
    return (lz_status)lz::set_last_error(LZ_ERR_TIMEOUT, msg);
  }
  lz::set_last_error(LZ_OK, "");
  return LZ_OK;
}

namespace {

// The failure path on purpose: an mbarrier that nothing arrives on.  The
// bounded wait gives up after its time limit, counts itself in the status
// word and the kernel returns; no fault, no hang.
__global__ void bounded_wait_selftest_kernel(unsigned int* status) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = lz::smem_u32(&bar);
  if (threadIdx.x == 0) {
    lz::mbar_init(b, 1);
    lz::mbar_init_fence();
  }
  __syncthreads();
  if (threadIdx.x == 0) lz::mbar_wait(b, 0, status);
}

}  // namespace

extern "C" lz_status lz_selftest_bounded_wait(lz_stream stream) {
  unsigned int* word = lz::device_status_word();
  if (word == nullptr)
    return (lz_status)lz::set_last_error(LZ_ERR_CUDA, "lz_selftest_bounded_wait: no device status word");
  bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(word);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    char msg[256];
    std::snprintf(msg, sizeof(msg), "lz_selftest_bounded_wait: %s", cudaGetErrorString(e));
    return (lz_status)lz::set_last_error(LZ_ERR_CUDA, msg);
  }
  lz::set_last_error(LZ_OK, "");
  return LZ_OK;
}
