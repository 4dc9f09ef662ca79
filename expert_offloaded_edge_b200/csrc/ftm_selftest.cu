// Failure-detection self-test of the bounded mbarrier wait the tensor-core
// kernels use: one thread waits on a barrier that nothing completes.  The wait
// gives up after kWaitLimitNs, records kDevErrTimeout in the device status
// word and returns false, and the kernel exits normally.
#include "ftm_common.cuh"

namespace ftm {

__global__ void wait_selftest_kernel() {
  __shared__ __align__(8) uint64_t never;
  if (threadIdx.x == 0) {
    mbar_init(&never, 1);   // one arrival expected; none ever comes
    fence_mbar_init();
    (void)mbar_wait(&never, 0u);
  }
}

cudaError_t launch_wait_selftest(cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>();
  return count_launch(cudaGetLastError());
}

}  // namespace ftm
