// selftest.cu -- a check of the bounded-wait machinery on the GPU: one CTA waits on
// an mbarrier phase that nothing completes, through the same wait_bounded() every
// pipeline wait of the library uses.  After the time limit the wait must give up,
// raise FA_DEV_WAIT_TIMEOUT in the device status word and return, leaving the
// context usable.  Nothing faults, traps or spins without a limit.
#include <cuda_runtime.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

__global__ void wait_timeout_selftest_kernel(unsigned int* status, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival completes phase 0; none ever comes
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtx w{&abort_flag, status, timeout_ns};
    wait_bounded(&bar, 0, w);
  }
}

cudaError_t launch_wait_timeout_selftest(unsigned int* status, uint64_t timeout_ns,
                                         cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace fa
