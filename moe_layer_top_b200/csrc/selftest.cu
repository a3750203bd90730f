// Failure-detection self-test: a kernel whose only wait can never complete.
//
// It initialises an mbarrier that nothing arrives at and waits on it through
// the same bounded wait (mbar_wait) that every pipeline kernel uses, with a
// caller-chosen limit.  The wait gives up, records the timeout code in the
// status word and the kernel returns normally, so the test shows -- without
// faulting, trapping or hanging the GPU -- that a stuck pipeline ends with an
// error status and leaves the context usable.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kWhereSelftest = 0x7F;

__global__ void bounded_wait_selftest_kernel(int* status, unsigned long long timeout_ns,
                                             unsigned long long* waited_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer_ns();
    const bool ok = mbar_wait(&bar, 0, &abort_flag, status, MOE_STATUS_WAIT_TIMEOUT | kWhereSelftest, timeout_ns);
    *waited_ns = globaltimer_ns() - t0;
    if (ok) report_status(status, -1);  // cannot happen: nothing arrives
  }
}

}  // namespace

cudaError_t launch_wait_selftest(int* status, unsigned long long timeout_ns, unsigned long long* waited_ns,
                                 cudaStream_t stream) {
  bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(status, timeout_ns, waited_ns);
  return cudaGetLastError();
}

}  // namespace moe
