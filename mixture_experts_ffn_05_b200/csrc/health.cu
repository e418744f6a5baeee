// Self-test of the device failure path.  Every kernel of the library bounds its waits on
// shared-memory barriers; a wait that runs out writes MOE_ERR_DEVICE_TIMEOUT into the
// workspace's status word and the kernel winds down instead of hanging.  This kernel runs
// one such bounded wait on a barrier that nothing ever completes, so a caller (or a test)
// can check that path end to end without faulting or hanging the GPU.
#include "common.cuh"
#include "internal.h"

namespace moe {

__global__ void __launch_bounds__(32) wait_selftest_kernel(unsigned* status, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival expected; none ever comes
    mbar_fence_init();
  }
  __syncwarp();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, timeout_ns, nullptr))
    record_status(status, kStatusTimeout);
}

cudaError_t launch_wait_selftest(unsigned* status, uint64_t timeout_ns, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace moe
