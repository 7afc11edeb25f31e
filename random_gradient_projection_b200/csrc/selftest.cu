// Self-test of the bounded mbarrier waits that every tensor-core kernel of the step uses
// (grape_selftest_wait_timeout).  One CTA waits on two mbarriers that nothing ever arrives
// on: warp 0 must give up at its own short limit and raise the CTA's abort flag, and
// warp 1, with a long limit, must leave early on that flag.  Nothing faults or hangs.
#include <cuda_runtime.h>

#include <cstdint>

#include "tc.h"
#include "tc_ptx.cuh"

namespace grape {

namespace {
__global__ void __launch_bounds__(64) wait_selftest_kernel(uint64_t short_ns, uint64_t long_ns, int* bits) {
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ int abort_word;
  if (threadIdx.x == 0) {
    abort_word = 0;
    ptx::mbar_init(&bar[0], 1);   // nothing ever arrives on either barrier
    ptx::mbar_init(&bar[1], 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort_flag = &abort_word;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane != 0) return;
  if (warp == 0) {
    // gives up at its own (short) limit and raises the CTA's abort flag
    if (!ptx::mbar_wait_or_abort(&bar[0], 0, short_ns, abort_flag)) atomicOr(bits, 1);
  } else {
    // the long limit must not be reached: the abort flag ends this wait first
    const uint64_t t0 = ptx::globaltimer_ns();
    if (!ptx::mbar_wait_or_abort(&bar[1], 0, long_ns, abort_flag))
      atomicOr(bits, (ptx::globaltimer_ns() - t0 < long_ns) ? 2 : 4);
  }
}
}  // namespace

cudaError_t tc_selftest_wait(uint64_t short_ns, uint64_t long_ns, int* bits_dev, cudaStream_t st) {
  wait_selftest_kernel<<<1, 64, 0, st>>>(short_ns, long_ns, bits_dev);
  return cudaGetLastError();
}

}  // namespace grape
