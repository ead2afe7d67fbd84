// velox_wait_selftest: the bounded waits of the library, driven to their limit.
//
// Every kernel that waits on an mbarrier (the attention CTAs' TMA, MMA and
// softmax roles) uses mbar_wait: a try-wait loop bounded by %globaltimer
// that, on giving up, sets a CTA-wide abort flag so that the CTA's other
// waiters stop too, and leaves the error to be reported through dev_status.
// This kernel runs exactly that code on barriers that nothing completes, so
// a test can watch the limit end the wait and the abort flag end the other
// waiters, with no fault, trap or hang.  It has no counterpart on the pages.
#include "common.cuh"

namespace velox {
namespace {

__global__ void __launch_bounds__(64) wait_selftest_kernel(uint64_t limit_ns,
                                                           int32_t *dev_status,
                                                           int64_t *elapsed_ns) {
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ int s_abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);  // nothing ever arrives on either barrier
    mbar_init(&bar[1], 1);
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int *abort = &s_abort;
  const uint64_t t0 = global_timer_ns();
  bool waited = false, ok = true;
  if (warp == 0) {
    if (lane == 0) {
      waited = true;
      ok = mbar_wait(&bar[0], 0, abort, limit_ns);
    }
  } else {
    // ten times the limit of its own: only the abort flag set by thread 0
    // can end this wait at about limit_ns
    waited = true;
    ok = mbar_wait(&bar[1], 0, abort, 10 * limit_ns);
  }
  const uint64_t t1 = global_timer_ns();
  if (waited && !ok && lane == 0) flag_error(dev_status, VELOX_DEV_WAIT_TIMEOUT);
  if (elapsed_ns && lane == 0) elapsed_ns[warp] = static_cast<int64_t>(t1 - t0);
}

}  // namespace

cudaError_t launch_wait_selftest(uint64_t limit_ns, int32_t *dev_status, int64_t *elapsed_ns,
                                 cudaStream_t stream) {
  wait_selftest_kernel<<<1, 64, 0, stream>>>(limit_ns, dev_status, elapsed_ns);
  return cudaGetLastError();
}

}  // namespace velox
