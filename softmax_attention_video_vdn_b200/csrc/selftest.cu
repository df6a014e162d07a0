// selftest.cu - exercises the bounded-wait failure path of the pipelines.
// A kernel waits on an mbarrier that nothing arrives on; the wait must give
// up after the given time, record VDN_ERR_TIMEOUT in the status word and let
// the kernel exit normally, leaving the CUDA context usable.
#include "kernels.h"

namespace vdn {

__global__ void wait_timeout_kernel(int32_t* dev_status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_sh;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const Abort ab{&abort_sh, dev_status};
  // no thread ever arrives on `bar`: every lane's wait ends by the limit
  (void)mbar_wait_limit(&bar, 0, ab, limit_ns);
  __syncthreads();
}

cudaError_t launch_wait_timeout(int32_t* dev_status, int limit_ms, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(dev_status, (uint64_t)limit_ms * 1000000ull);
  return cudaGetLastError();
}

}  // namespace vdn
