// selftest.cu -- the bounded-wait failure path, exercised on purpose.
//
// Every wait of the library's kernels (on a TMA completion or on another
// warp's arrival) gives up after a time limit, sets PKV_STATUS_WAIT_TIMEOUT
// and lets the kernel return, so that a lost arrival shows up as a status bit
// instead of a hung GPU.  This kernel makes that path run: one thread
// initialises an mbarrier that nothing ever arrives on and waits for it with
// mbar_wait_bounded -- the helper every kernel uses -- and a short limit.  No
// copy or MMA is ever started, so nothing is in flight when it gives up.
#include "common.cuh"
#include "launch.h"

namespace pkv {

__global__ void __launch_bounds__(32) wait_timeout_selftest_kernel(unsigned* status, uint64_t limit_ns,
                                                                    unsigned* gave_up) {
  pdl_wait_and_release();
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_barrier_init();
  }
  __syncwarp();
  // every lane waits (as a warp does in the kernels); the phase never completes
  const bool ok = __all_sync(kFullMask, mbar_wait_bounded(b, 0, status, limit_ns));
  if (threadIdx.x == 0) *gave_up = ok ? 0u : 1u;
}

cudaError_t launch_wait_timeout_selftest(unsigned* status, uint64_t limit_ns, unsigned* gave_up, cudaStream_t st) {
  return launch_pdl(wait_timeout_selftest_kernel, dim3(1), dim3(32), 0, st, status, limit_ns, gave_up);
}

}  // namespace pkv
