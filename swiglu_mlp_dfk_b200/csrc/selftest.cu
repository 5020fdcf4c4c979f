// selftest.cu -- a self-test of the failure detection every pipeline kernel
// relies on: a bounded mbarrier wait that nothing ever completes must give
// up after the device's wait limit, record the timeout in the device status
// block and let the kernel return, leaving the context usable.  No fault,
// trap or endless loop is involved: the wait is the same bounded wait the
// weight-streaming kernels use.
#include <cuda_runtime.h>

#include "launch_util.h"
#include "ptx.cuh"

namespace dfk {

__global__ void __launch_bounds__(32) wait_selftest_kernel(unsigned *err,
                                                           unsigned long long *elapsed_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival expected; none is ever made
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    const unsigned long long t0 = global_timer_ns();
    // phase 0 of a fresh barrier completes only after an arrival
    const bool done = mbar_wait_bounded(&bar, 0, &abort_flag, err);
    *elapsed_ns = done ? 0ull : global_timer_ns() - t0;
  }
}

cudaError_t launch_wait_selftest(unsigned *err, unsigned long long *elapsed_ns, cudaStream_t s) {
  void *args[] = {&err, &elapsed_ns};
  return launch_kernel(reinterpret_cast<const void *>(&wait_selftest_kernel), dim3(1), dim3(32),
                       0, s, false, args);
}

}  // namespace dfk
