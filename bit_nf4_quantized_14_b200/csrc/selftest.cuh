// Self-test of the bounded waits: a one-warp kernel waits on something that never happens -- an
// mbarrier no thread arrives on, or a device word nothing writes -- and must give up after the wait
// limit in force, record QLORA_STATUS_TIMEOUT in the status word and return, leaving the context usable.
// Nothing here faults, traps or spins without a bound.
#pragma once

#include "common.cuh"

namespace qnf4 {

__device__ uint64_t g_selftest_word;   // stays 0; the word wait below wants ~0

__global__ void __launch_bounds__(32) bounded_wait_selftest_kernel(int kind) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (kind == 0)
    (void)mbar_wait(&bar, 0);                          // phase 0 never completes: count 1, no arrival
  else
    (void)wait_word_eq(&g_selftest_word, ~0ull);
}

}  // namespace qnf4
