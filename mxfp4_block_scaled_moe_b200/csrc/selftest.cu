// Self-test of the bounded device wait (mxmoe_selftest_wait_timeout): one thread waits,
// through the same mbar_wait the tensor-core kernels use, on an mbarrier that nothing
// completes, so the wait expires, sets MXMOE_ETIMEOUT in the error word and returns.
#include "launchers.h"
#include "tc_common.cuh"

namespace mxmoe {

namespace {

__global__ void __launch_bounds__(32) wait_selftest_kernel(int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_word;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);   // expects one arrival that never comes
    abort_word = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  __syncwarp();
  if (threadIdx.x == 0) tc::mbar_wait(&bar, 0, &abort_word, err);
}

}  // namespace

cudaError_t launch_wait_selftest(int* err, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(err);
  return cudaGetLastError();
}

}  // namespace mxmoe
