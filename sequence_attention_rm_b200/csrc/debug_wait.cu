// Test hook for the bounded-wait machinery: one CTA waits on an mbarrier that
// nothing arrives at, gives up after `spin_limit` polls and records a timeout
// in the device status word.  Nothing faults and nothing hangs.
#include "internal.h"
#include "tc_common.cuh"

namespace rm {

namespace {
__global__ void expire_wait_kernel(uint32_t spin_limit, unsigned int* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t polls = 0;
    while (!tc::mbar_try_wait(&bar, 0)) {
      if (++polls >= spin_limit) {
        report_timeout(status);
        break;
      }
    }
  }
}
}  // namespace

cudaError_t launch_debug_expire_wait(uint32_t spin_limit, unsigned int* status,
                                     cudaStream_t stream) {
  expire_wait_kernel<<<1, 32, 0, stream>>>(spin_limit, status);
  return cudaGetLastError();
}

}  // namespace rm
