// selftest.cuh - self-test of the failure path of the grouped GEMM's waits.
#pragma once
#include "ptx.cuh"

namespace moe {

// Diagnostic of the bounded wait: one thread waits, through mbar_wait, on the
// first phase of a fresh mbarrier that nothing arrives on. After
// kWaitTimeoutNs the wait records kErrWaitTimeout and the kernel returns; it
// touches only its own shared memory and the error word.
__global__ void k_selftest_wait_timeout() {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
    mbar_wait(&bar, 0, &abort_flag);  // phase 0 never completes
  }
}

}  // namespace moe
