// fa_selftest.cuh - a kernel that exercises the bounded waits of the library
// on purpose, so that the timeout path can be tested on a GPU without any
// fault or hang.
//
// Two warps of one CTA wait on mbarriers that nothing ever arrives on, with
// the same mbar_wait/Watchdog code as the attention kernels.  Warp 0 waits
// with a short limit: when it expires, it records kDevErrTimeout in the
// library's error flag and marks the CTA aborted.  Warp 1 waits with the
// kernels' own 4 s limit and must leave as soon as it sees the abort mark,
// which is how every role of an attention kernel leaves once one role gives
// up.  The kernel then returns normally; the host reads the flag.
#pragma once

#include "sm100.cuh"

namespace fa {

__global__ void __launch_bounds__(64, 1) fa_watchdog_selftest_kernel(int* dev_error, uint64_t timeout_ns) {
  __shared__ uint64_t bar[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const Watchdog wd{&abort_flag, dev_error};
  const int warp = int(threadIdx.x >> 5);
  if (lane_id() == 0) {
    if (warp == 0)
      mbar_wait(&bar[0], 0, wd, timeout_ns);   // expires after timeout_ns
    else
      mbar_wait(&bar[1], 0, wd);               // leaves on the abort mark
  }
  __syncwarp();
  __syncthreads();
}

}  // namespace fa
