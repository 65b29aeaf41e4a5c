// Self-test of the bounded waits that every kernel of this library uses on its mbarriers
// (wait_bar in sm100_ptx.cuh): thread 0 of one CTA waits on a barrier that nothing ever arrives
// at.  After the bound the wait gives up, sets the CTA's abort flag, ORs the timeout bit into
// the device status word and returns, and the kernel exits: no hang, no fault, and the next
// attn_device_status() reports ATTN_ERR_TIMEOUT with the context still usable.

#include "attn_selftest.h"
#include "sm100_ptx.cuh"

namespace ea {

namespace {

__global__ void __launch_bounds__(32) wait_selftest_kernel(int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    bar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const AbortState ab{&abort_flag, status};
    wait_bar(&bar, 0, ab);  // phase 0 never completes: no thread arrives
  }
}

}  // namespace

cudaError_t launch_wait_selftest(int* status, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(status);
  return cudaGetLastError();
}

}  // namespace ea
