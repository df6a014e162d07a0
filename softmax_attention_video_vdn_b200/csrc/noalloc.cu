// noalloc.cu - vda_bidir_scan_noalloc: the bidirectional scan for callers
// that cannot allocate device memory at call time (for example code that runs
// inside another framework's allocator or plugin hook, or a real-time loop
// that forbids allocation). The scan's scratch (the per-frame maps A_f, B_f)
// lives in a fixed array inside the library instead of a caller workspace.
#include <stdio.h>

#include <mutex>

#include "kernels.h"

namespace vdn {

// Scratch of the no-allocation scan. With CUDA's lazy module loading (the
// default) a device holds these 16 MiB from the first call that looks up its
// address there (with CUDA_MODULE_LOADING=EAGER, from the moment the library
// is loaded) until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_scan_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
std::mutex g_scratch_mu;
// Per device: the ID of the context the address was looked up in (context
// IDs are never reused within a process; 0 = none yet), and the address.
unsigned long long g_scratch_ctx[kMaxDevices] = {};
void* g_scratch_ptr[kMaxDevices] = {};

void* driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return p;
}

// ID of the context bound to the calling thread; 0 if there is none.
bool current_ctx_id(unsigned long long* id) {
  static CtxGetCurrentFn get = reinterpret_cast<CtxGetCurrentFn>(driver_fn("cuCtxGetCurrent"));
  static CtxGetIdFn get_id = reinterpret_cast<CtxGetIdFn>(driver_fn("cuCtxGetId"));
  if (!get || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return false;
  *id = 0;
  return !ctx || get_id(ctx, id) == CUDA_SUCCESS;
}
}  // namespace

// Device address of g_scan_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// the device current and cached together with the ID of the context it
// belongs to. A
// device reset (cudaDeviceReset) or a destroyed and recreated primary context
// gives the device a new context, and with it a new lookup, so a stale
// address from the old context is never handed to a kernel.
cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  // No context bound to this thread yet reads as ID 0 and never matches the
  // cache; cudaGetSymbolAddress then binds the device's primary context.
  unsigned long long id = 0;
  if (!current_ctx_id(&id)) return cudaErrorInitializationError;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (id == 0 || g_scratch_ctx[dev] != id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scan_scratch);
    if (e != cudaSuccess) return e;
    if (!current_ctx_id(&id) || id == 0) return cudaErrorInitializationError;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = id;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

}  // namespace vdn
