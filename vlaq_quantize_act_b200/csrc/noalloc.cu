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
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"

namespace vlaq {

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

namespace {

std::mutex g_mu;
// per device: the address of the array and the context it was resolved in
struct Resolved {
  unsigned long long ctx_id;
  void* ptr;
};
Resolved g_res[kMaxDevices] = {};

// Identity of the current context: the driver's context ID, unique for the
// life of the process (a context created after cudaDeviceReset gets a new
// one even if its handle value is reused); the handle value where the
// driver has no context IDs.  0 if no context is current.
unsigned long long current_context_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  if (!get_current || get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  unsigned long long id = 0;
  if (get_id && get_id(ctx, &id) == CUDA_SUCCESS) return id + 1;  // never 0
  return static_cast<unsigned long long>(reinterpret_cast<uintptr_t>(ctx));
}

}  // namespace

// Device address of the scratch array in the current device's context.
// The first call in a context (with that device current) resolves it with
// cudaGetSymbolAddress and caches it beside the context's identity; later
// calls in the same context only read the cache, and a call in a new
// context (after cudaDeviceReset, say) resolves it again.
cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* p = nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  unsigned long long id = current_context_id();
  if (!g_res[dev].ptr || id == 0 || g_res[dev].ctx_id != id) {
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (id == 0) id = current_context_id();  // the lookup made the primary context current
    g_res[dev].ctx_id = id;
    g_res[dev].ptr = p;
  }
  *out = g_res[dev].ptr;
  return cudaSuccess;
}

// Zeroes the scratch array of the current device on stream s, if a call has
// resolved it in the current context (an array no call has used in this
// context is still zero from the module load).
cudaError_t noalloc_clear(cudaStream_t s) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaSuccess;
  void* p = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    const unsigned long long id = current_context_id();
    if (id != 0 && g_res[dev].ctx_id == id) p = g_res[dev].ptr;
  }
  return p ? cudaMemsetAsync(p, 0, kNoallocScratchBytes, s) : cudaSuccess;
}

}  // namespace vlaq
