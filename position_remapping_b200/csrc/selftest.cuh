// Failure-detection self-test: one CTA waits on an mbarrier that nothing
// completes, with a short limit, and gives up through the same bounded wait
// that every kernel of the library uses (device status word set, wait
// abandoned, kernel returns). No fault, trap or endless loop is involved;
// the context stays usable.
#pragma once

#include "common.cuh"

namespace ropeattn {

__global__ void wait_selftest_kernel(unsigned long long limit_ns, int* result) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);          // one arrival expected; none is ever made
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) *result = mbar_wait(&bar, 0, &abort_flag, limit_ns) ? 1 : 0;
}

}  // namespace ropeattn
