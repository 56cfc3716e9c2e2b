// selftest.cu -- exercises the failure path every bounded device-side wait of
// the library shares, without faulting anything: one CTA waits on an mbarrier
// that nothing completes; the wall-clock bound (kWaitLimitNs) runs out, the
// wait records kErrTimeout in the device error word and the kernel returns.
#include "nf4_common.cuh"
#include "internal.h"

namespace nf4 {
namespace {

__global__ void wait_timeout_kernel(unsigned* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // expects one arrival that never comes
    fence_mbar_init();
    mbar_wait_bounded(&bar, 0, err);
  }
}

}  // namespace

cudaError_t launch_wait_timeout(unsigned* err, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(err);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace nf4
