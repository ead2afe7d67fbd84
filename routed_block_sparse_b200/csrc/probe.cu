// velox_clock_probe: the SM clock seen from inside the GPU, for measurement.
//
// The B200's power limiter can hold the SM clock well below what the
// driver's sampled clock reports while a heavy kernel runs.  This one-CTA
// kernel samples the SM cycle counter (clock64) against the global
// nanosecond timer (%globaltimer) at a fixed pause; run beside another
// kernel on its own stream (it needs one warp, no shared memory and a few
// registers, so it fits on an SM next to that kernel's CTA), the ratio of
// successive samples is the SM clock during that kernel.  It has no
// counterpart on the pages.
#include "common.cuh"

namespace velox {
namespace {

__global__ void __launch_bounds__(32) clock_probe_kernel(int64_t *samples, int n,
                                                         uint32_t pause_ns) {
  if (threadIdx.x != 0) return;
  for (int k = 0; k < n; ++k) {
    const uint64_t t = global_timer_ns();
    samples[2 * k] = static_cast<int64_t>(clock64());
    samples[2 * k + 1] = static_cast<int64_t>(t);
    __nanosleep(pause_ns);
  }
}

}  // namespace

cudaError_t launch_clock_probe(int64_t *samples, int n, uint32_t pause_ns, cudaStream_t stream) {
  clock_probe_kernel<<<1, 32, 0, stream>>>(samples, n, pause_ns);
  return cudaGetLastError();
}

}  // namespace velox
