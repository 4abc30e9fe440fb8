// lz_swa_meta_bwd_noalloc: the window + meta-token backward for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they run the
// backward: an inference or training engine whose plugin hook must not
// allocate while it enqueues work, or a host framework that has already
// reserved all device memory for its own pool.  They cannot supply the
// scratch that lz_swa_meta_bwd asks for, so this entry point uses a fixed
// scratch array compiled into the library instead.
//
// The array below lives in device memory of every GPU that loads the
// library, for the life of the process.  In host code its name is only a
// host-side stand-in, not a device address, so the address passed to the
// kernels is looked up once per device with cudaGetSymbolAddress, with that
// device current.
#include <cstdio>
#include <mutex>
#include <unordered_map>

#include "../../include/lizard.h"
#include "kernels.h"

namespace lz {
// The window entry points' checks of a dims struct (lizard_api.cu): LZ_OK, or
// the status they return, with the error recorded.
int check_window_dims(const lz_dims* d);
}  // namespace lz

namespace {

constexpr size_t kScratchBytes = LZ_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_swa_bwd_scratch[kScratchBytes];

std::mutex g_mu;
std::unordered_map<int, void*> g_addr;  // device ordinal -> device address of the array

}  // namespace

extern "C" lz_status lz_swa_meta_bwd_noalloc(const lz_dims* d, const void* q, const void* k,
                                            const void* v, const void* meta_k,
                                            const void* meta_v, const float* lse,
                                            const void* o, const void* dO, void* dq,
                                            void* dk, void* dv,
                                            float* dmeta_k, float* dmeta_v, lz_stream stream) {
  // shapes first, so that a bad call touches no device state
  const int chk = lz::check_window_dims(d);
  if (chk != LZ_OK) return (lz_status)chk;
  const size_t need = lz_workspace_bytes(d, LZ_WS_SWA_BWD);
  if (need > kScratchBytes) {
    char msg[256];
    std::snprintf(msg, sizeof(msg),
                  "lz_swa_meta_bwd_noalloc: problem needs %zu bytes of scratch, more than the "
                  "%zu-byte static array; use lz_swa_meta_bwd with caller-owned scratch",
                  need, kScratchBytes);
    return (lz_status)lz::set_last_error(LZ_ERR_UNSUPPORTED, msg);
  }
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    char msg[256];
    std::snprintf(msg, sizeof(msg), "lz_swa_meta_bwd_noalloc: cudaGetDevice: %s",
                  cudaGetErrorString(e));
    return (lz_status)lz::set_last_error(LZ_ERR_CUDA, msg);
  }
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = g_addr.find(dev);
    if (it == g_addr.end()) {
      // First call on this device: look up the array's device address.  With
      // lazy module loading (the CUDA 12 default) this is also where the
      // module, and with it the 16 MiB array, is loaded onto the device, so it
      // can fail if the device's memory is exhausted, and it must not happen
      // inside a stream capture.  The address stays valid until the process
      // exits or the device is reset (cudaDeviceReset unloads the module:
      // after that this entry point must not be used in the process).
      e = cudaGetSymbolAddress(&scratch, g_swa_bwd_scratch);
      if (e != cudaSuccess || scratch == nullptr) {
        char msg[256];
        std::snprintf(msg, sizeof(msg),
                      "lz_swa_meta_bwd_noalloc: cudaGetSymbolAddress on device %d: %s", dev,
                      cudaGetErrorString(e));
        return (lz_status)lz::set_last_error(LZ_ERR_CUDA, msg);
      }
      g_addr.emplace(dev, scratch);
    } else {
      scratch = it->second;
    }
  }
  // Every region of this scratch is written before it is read, so the
  // previous call's leftovers need no clearing.
  return lz_swa_meta_bwd(d, q, k, v, meta_k, meta_v, lse, o, dO, dq, dk, dv, dmeta_k, dmeta_v,
                         scratch, kScratchBytes, stream);
}
