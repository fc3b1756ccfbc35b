// selftest.cu -- a diagnostic launch that exercises the bounded device waits
// every kernel of the library uses, without faulting, trapping or hanging.
//
// One CTA runs two of the bounded waits and writes their results to out[0],
// out[1].  mode 1: thread 0 arrives on an mbarrier first, then waits on its
// phase with mbar_wait_guarded (the wait the pipelines use) and
// mbar_wait_backoff (the epilogue's); both succeed.  mode 0: nothing arrives;
// the first wait gives up after `budget` SM cycles, ORs STRATA_DEV_TIMEOUT
// into the status word and raises the CTA's abort flag, and the second
// returns at once because of that flag.  mode 2: the first wait is
// gmem_wait_geq (the fused decode kernel's wait on a counter other CTAs
// raise) on out[0], zeroed first and raised by nobody; it gives up the same
// way, and the mbarrier wait after it returns at once.
#include "decode.cuh"
#include "tc05.cuh"

namespace strata {

__global__ void __launch_bounds__(32, 1)
wait_selftest_kernel(long long budget, int mode, int32_t* status, int32_t* out) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    bool ok1;
    if (mode == 2) {
      out[0] = 0;
      __threadfence();
      ok1 = gmem_wait_geq(out, 1, status, &abort_flag, budget);
    } else {
      if (mode == 1) mbar_arrive(&bar);
      ok1 = mbar_wait_guarded(&bar, 0, status, &abort_flag, budget);
    }
    const bool ok2 = mbar_wait_backoff(&bar, 0, status, &abort_flag, budget);
    out[0] = ok1 ? 1 : 0;
    out[1] = ok2 ? 1 : 0;
  }
}

cudaError_t launch_wait_selftest(long long budget, int mode, int32_t* status, int32_t* out,
                                 cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(budget, mode, status, out);
  return cudaGetLastError();
}

}  // namespace strata
