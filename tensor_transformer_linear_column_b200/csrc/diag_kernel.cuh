// diag_kernel.cuh -- a kernel that makes the library's bounded wait run out on
// purpose, so the timeout path (error word, abort flag shared by the roles of a
// CTA, host-side report and clearing) can be tested without a fault or a hang.
#pragma once

#include "ptx.cuh"

namespace tpb {

// One CTA of two warps.  Each waits, through wait_parity, on its own mbarrier
// that nothing ever arrives on: lane 0 of warp 0 with a limit of `limit_ns`,
// lane 0 of warp 1 with the library's default limit.  Warp 0's wait runs out,
// records kErrTimeout in g_tp_device_error and raises the CTA's abort flag;
// warp 1's wait must then return false within a few polls instead of running
// to its own limit.  result[0], result[1]: what the two waits returned (1 =
// phase completed, 0 = gave up); result[2]: nanoseconds warp 1 waited.
__global__ void __launch_bounds__(64, 1)
    bounded_wait_probe_kernel(unsigned long long limit_ns, int* result) {
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars[0]), 1);
    mbar_init(smem_u32(&bars[1]), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort = &abort_flag;
  if (threadIdx.x == 0) {
    result[0] = wait_parity(smem_u32(&bars[0]), 0u, abort, limit_ns) ? 1 : 0;
  } else if (threadIdx.x == 32) {
    const unsigned long long t0 = globaltimer_ns();
    result[1] = wait_parity(smem_u32(&bars[1]), 0u, abort) ? 1 : 0;
    const unsigned long long waited = globaltimer_ns() - t0;
    result[2] = waited > 0x7fffffffull ? 0x7fffffff : static_cast<int>(waited);
  }
}

}  // namespace tpb
