// noalloc.cu - vda_bidir_scan_noalloc: the bidirectional scan for callers
// that cannot allocate device memory at call time (for example code that runs
// inside another framework's allocator or plugin hook, or a real-time loop
// that forbids allocation). The scan's scratch (the per-frame maps A_f, B_f)
// lives in a fixed array inside the library instead of a caller workspace.
#include <stdio.h>

#include <mutex>

#include "kernels.h"

namespace vdn {

// Scratch of the no-allocation scan. Every GPU that loads the library holds
// these 16 MiB until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_scan_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};
}  // namespace

// Device address of g_scan_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scan_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

}  // namespace vdn
