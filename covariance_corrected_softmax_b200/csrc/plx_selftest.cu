// plx_selftest.cu -- failure-detection self-test: a kernel whose one wait can
// never be satisfied, so that the bounded wait every kernel of the library uses
// (mbar_wait) runs out of time, records kDevTimeoutMbarrier in the device
// status block and returns.  The pages have no counterpart to this: it checks
// the library's own promise that no kernel waits forever.
#include "plx_launch.h"

namespace plx {

__global__ void __launch_bounds__(32, 1) plx_selftest_wait_kernel(unsigned* err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);  // one arrival expected; none ever comes
    fence_mbarrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    // Phase 0 never completes: the wait ends by its wall-clock limit (or, should
    // the clock stop, its poll backstop), recording the timeout.
    const bool ok = mbar_wait(&bar, 0, reinterpret_cast<volatile int*>(&abort_flag), err);
    if (ok) record_error(err, kDevBadArgument);  // an impossible completion
  }
  __syncwarp();
}

cudaError_t launch_selftest_wait(unsigned* err, cudaStream_t stream) {
  plx_selftest_wait_kernel<<<1, 32, 0, stream>>>(err);
  return cudaGetLastError();
}

}  // namespace plx
