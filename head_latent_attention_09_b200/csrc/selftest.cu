// Self-test of the device-side time-out path.  Every wait in the library's
// kernels polls an mbarrier phase against %globaltimer and, past its limit,
// sets the status word's time-out bit and gives up instead of hanging.  This
// kernel runs one such wait on a barrier that nothing ever completes, with a
// short limit, so that a test can watch the path end in MLA_ERR_TIMEOUT with
// the context still usable afterwards.  It touches no memory but its own
// shared barrier and the status word.
#include "ptx.cuh"

namespace mla {
namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(unsigned *status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);   // one arrival completes phase 0; none is ever made
    ptx::fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x != 0) return;
  const unsigned long long t0 = ptx::globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (ptx::mbar_test_wait(&bar, 0)) return;   // cannot happen: nobody arrives
    if ((i & 63u) == 0 && ptx::globaltimer() - t0 > limit_ns) {
      atomicOr(status, kStatusTimeout);
      return;
    }
  }
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(unsigned *status, unsigned long long limit_ns, cudaStream_t s) {
  wait_timeout_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace mla
