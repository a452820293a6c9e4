// Failure-detection self test: a block waits with the library's bounded
// wait on a barrier that nothing completes.  The wait must give up after
// `cap` polls and record kStatusWaitCap; the block then returns normally.
#include "fvattn_internal.cuh"

namespace fvattn {

__global__ void wait_selftest_kernel(int* status, long long cap) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, status, cap);
}

cudaError_t launch_wait_selftest(int* status, long long cap, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(status, cap);
  return cudaGetLastError();
}

}  // namespace fvattn
