// selftest.cu -- a check of the failure-detection path itself: one thread waits, through the
// same bounded wait every kernel uses, on a shared-memory mbarrier that nothing arrives on.
// The wait runs out after its limit, records kErrWaitSelftest in the device error word and
// returns, so the kernel ends normally and the context stays usable.
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace qlora {

namespace {

__global__ void bounded_wait_selftest_kernel(int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0u, kErrWaitSelftest, err, 0);
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(int* err, cudaStream_t stream) {
  bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(err);
  return cudaGetLastError();
}

}  // namespace qlora
