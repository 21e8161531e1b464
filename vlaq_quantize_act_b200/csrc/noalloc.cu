// Scratch memory for vlaq_linear_nvfp4_noalloc: a fixed device array that
// lives in the library image, so callers that must not allocate device
// memory can still run the split-K path of the NVFP4 linear.
//
// Who needs this: code that runs where cudaMalloc is off limits, for
// example inside a host callback, from a real-time control loop that must
// not take the allocator's locks or risk an allocation failure mid-episode,
// or in an embedding that owns all device memory through its own arena and
// forbids other allocations.  Such callers pass inputs and outputs only.
//
// The array is a module global: every GPU that loads the library holds it
// (kNoallocScratchBytes) until the process exits.  All calls on a device
// share it.  It is zero when the module loads and the GEMM leaves its
// split-K tile counters zero after every call; after a timed-out call
// vlaq_check clears it (noalloc_clear).  Calls that overlap on the GPU
// (different streams, or different host threads) race on it.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"

namespace vlaq {

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

namespace {
std::mutex g_mu;
void* g_ptr[kMaxDevices] = {nullptr};
}  // namespace

// Device address of the scratch array on the current device.  The first
// call per device resolves it with cudaGetSymbolAddress (with that device
// current) and caches it; later calls only read the cache.
cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_ptr[dev] = p;
  }
  *out = g_ptr[dev];
  return cudaSuccess;
}

// Zeroes the scratch array of the current device on stream s (only if a
// call has resolved it on this device).
cudaError_t noalloc_clear(cudaStream_t s) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaSuccess;
  void* p = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    p = g_ptr[dev];
  }
  return p ? cudaMemsetAsync(p, 0, kNoallocScratchBytes, s) : cudaSuccess;
}

}  // namespace vlaq
