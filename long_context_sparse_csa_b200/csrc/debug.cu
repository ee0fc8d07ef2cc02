// Test aid: a kernel whose bounded wait runs out on purpose, so that the host can check the whole
// failure-reporting path (wait limit -> device error word -> csa_device_error) without a fault.
//
// The kernel initialises one mbarrier in shared memory, which nothing ever arrives on, and waits on
// its first phase with the library's bounded wait (the same helper every pipeline wait uses) and
// the caller's limit.  When the limit passes, thread 0 sets the timeout bit of the error word and
// the CTA returns: no copy, MMA or tensor memory is ever in flight in it.
#include "kernels.h"
#include "sm100.cuh"

namespace csa {

namespace {

__global__ void __launch_bounds__(32) wait_probe_kernel(int* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0 && !sm100::mbar_wait(&bar, 0u, limit_ns)) set_device_error(err, kErrWaitTimeout);
}

}  // namespace

cudaError_t launch_wait_probe(int* err, uint64_t limit_ns, cudaStream_t s) {
  return launch_kernel(wait_probe_kernel, dim3(1), dim3(32), 0, s, 0, err, limit_ns);
}

}  // namespace csa
