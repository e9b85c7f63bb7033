// Self-test of the bounded-wait path every libpa kernel uses (sm_100a).
//
// The kernels never wait without a limit: a wait on an mbarrier that does
// not complete in time gives up, records a timeout in the device error word
// and lets the kernel return, so the CUDA context stays usable and the host
// learns of it through pa_device_error.  This kernel exercises that path on
// purpose and safely: one CTA waits, with a short poll limit, on a barrier
// that nothing will ever complete, gives up and records the timeout.
#include "pa_device.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

__global__ void wait_timeout_selftest_kernel(uint32_t polls) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  // phase 0 of `bar` needs one arrival that never comes
  const bool done = mbar_wait_bounded(&bar, 0, polls);
  if (!done && threadIdx.x == 0) report_error(kErrTimeout);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(1u << 12);
  return cudaGetLastError();
}

}  // namespace pa
