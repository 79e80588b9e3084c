// Test hooks.  (1) The bounded-wait machinery: one CTA waits on an mbarrier
// that nothing arrives at, gives up after `spin_limit` polls and records a
// timeout in the device status word.  Nothing faults and nothing hangs.
// (2) The forward's polynomial exponential, evaluated on caller-given inputs
// so that a test can compare it with the exact 2^x over its input range.
#include "exp2_poly.cuh"
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

// y[i] = exp2_fma2(x[i]) for i < n, two elements per thread (the function
// works on pairs); an odd tail pairs the last element with itself.
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  const int64_t pairs = (n + 1) / 2;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < pairs;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t a = 2 * i, b = 2 * i + 1 < n ? 2 * i + 1 : 2 * i;
    const float2 r = exp2_fma2(make_float2(x[a], x[b]));
    y[a] = r.x;
    if (b != a) y[b] = r.y;
  }
}
}  // namespace

cudaError_t launch_debug_exp2_poly(const float* x, float* y, int64_t n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int64_t pairs = (n + 1) / 2;
  const int64_t blocks = (pairs + 255) / 256;
  exp2_poly_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, stream>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_debug_expire_wait(uint32_t spin_limit, unsigned int* status,
                                     cudaStream_t stream) {
  expire_wait_kernel<<<1, 32, 0, stream>>>(spin_limit, status);
  return cudaGetLastError();
}

}  // namespace rm
