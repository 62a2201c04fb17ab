// wait_selftest.cuh - failure-detection self-test for the bounded device waits.
//
// Every wait in the hs2 kernels (an mbarrier phase that a TMA copy, an MMA
// commit or another warp completes) spins for at most a fixed number of SM
// cycles; when the limit runs out the kernel records HS2_ERR_TIMEOUT in the
// device error word and winds down instead of hanging the GPU.  This kernel
// makes such a wait run out on purpose, with nothing that could ever end it,
// so that a test can check the whole chain: the wait gives up, the error word
// is set, the host reads it with hs2_get_last_device_error, and the context
// stays usable for the next launch.  Nothing faults: the wait is a plain
// bounded loop over try-wait / load, and the kernel touches no memory but its
// own shared barrier, a zero-initialised device word and the error word.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace hs2 {

// A device word that no code ever writes: the "flag that nothing sets".
__device__ int g_wait_selftest_flag = 0;

// mode 0: wait on phase 0 of a shared-memory mbarrier that expects one arrival
//         and never gets it (the form of every pipeline wait in the kernels).
// mode 1: wait for a global flag that no one sets (the form of a cross-CTA or
//         cross-rank flag wait).
// Either wait gives up after ``limit`` SM cycles and records HS2_ERR_TIMEOUT.
__global__ void __launch_bounds__(32) k_wait_selftest(int mode, long long limit, int* err) {
  grid_dep_wait();
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x != 0) return;
  const volatile int* flag = &g_wait_selftest_flag;
  const long long t0 = clock64();
  bool done = false;
  for (;;) {
    done = mode == 0 ? mbar_try_wait(&bar, 0) : (*flag != 0);
    if (done || clock64() - t0 > limit) break;
  }
  if (!done) record_error(err, HS2_ERR_TIMEOUT);
}

}  // namespace hs2
