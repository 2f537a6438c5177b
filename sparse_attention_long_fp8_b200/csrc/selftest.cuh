// Failure-detection self-test kernel: a bounded wait that nothing completes.
#pragma once

#include "ptx.cuh"

namespace dsa {

// Waits on an mbarrier that nothing ever arrives on: the bounded wait runs out
// after limit_ns, raises the timeout bit of the error word and the kernel
// returns normally.
__global__ void wait_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  mbar_wait_limit(&bar, 0, limit_ns);
  __syncthreads();
}

}  // namespace dsa
