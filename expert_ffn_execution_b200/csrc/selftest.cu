// selftest.cu -- a diagnostic launch that exercises the bounded device waits
// every kernel of the library uses, without faulting, trapping or hanging.
//
// One CTA initialises an mbarrier and waits on its first phase twice: first
// with mbar_wait_guarded (the wait the pipelines use), then with
// mbar_wait_backoff (the epilogue's).  With `complete` set, thread 0 arrives
// first, so both waits succeed; without it nothing ever arrives, the first
// wait gives up after `budget` SM cycles, ORs STRATA_DEV_TIMEOUT into the
// status word and raises the CTA's abort flag, and the second wait returns
// at once because of that flag.  out[0], out[1] receive the two results.
#include "decode.cuh"
#include "tc05.cuh"

namespace strata {

__global__ void __launch_bounds__(32, 1)
wait_selftest_kernel(long long budget, int complete, int32_t* status, int32_t* out) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    if (complete) mbar_arrive(&bar);
    const bool ok1 = mbar_wait_guarded(&bar, 0, status, &abort_flag, budget);
    const bool ok2 = mbar_wait_backoff(&bar, 0, status, &abort_flag, budget);
    out[0] = ok1 ? 1 : 0;
    out[1] = ok2 ? 1 : 0;
  }
}

cudaError_t launch_wait_selftest(long long budget, int complete, int32_t* status, int32_t* out,
                                 cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(budget, complete, status, out);
  return cudaGetLastError();
}

}  // namespace strata
