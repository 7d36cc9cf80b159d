// Self-test of the failure-detection path: a kernel waits on an mbarrier that nothing will
// complete, with a caller-given time limit, and must end by itself, recording DSA_ERR_TIMEOUT
// in the device error word (the same bounded-wait scheme every pipeline wait of the library
// uses, with a short limit so a test takes milliseconds).  No fault, trap or hang is involved:
// the kernel returns normally and the context stays usable.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dsa {

__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    dev::mbar_init(&bar, 1);  // expects one arrival; none will come
    dev::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t a = dev::smem_addr(&bar);
    const uint64_t t0 = dev::global_timer_ns();
    bool done = false;
    while (!done) {
      if (dev::mbar_test(a, 0u)) {
        done = true;
      } else if (dev::global_timer_ns() - t0 > limit_ns) {
        record_device_error(DSA_ERR_TIMEOUT);
        break;
      }
    }
  }
  __syncthreads();
}

}  // namespace dsa
