// selftest.cu -- exercises the library's bounded wait without any fault: one
// thread waits, through the same helper every counter barrier of the library
// uses, on a counter that nothing increments.  The wait must give up after
// its limit, raise the TIMEOUT flag in the status word and return, leaving
// the context usable.
#include "common.cuh"
#include "internal.h"

namespace sd {
namespace {

__global__ void selftest_wait_kernel(const uint32_t *ctr, uint64_t limit_ns, uint32_t *status) {
  if (threadIdx.x == 0) wait_counter_geq(ctr, 1u, limit_ns, status);
}

}  // namespace

cudaError_t launch_selftest_wait(uint32_t *ctr, uint64_t limit_ns, uint32_t *status,
                                 cudaStream_t st) {
  if (limit_ns > kWaitLimitNs) limit_ns = kWaitLimitNs;
  selftest_wait_kernel<<<1, 32, 0, st>>>(ctr, limit_ns, status);
  return cudaGetLastError();
}

}  // namespace sd
