// Self-test of the bounded device waits: one CTA waits on an mbarrier that nothing arrives
// on, with a short limit, so the wait expires the way a real one would (the CTA's abort flag
// set, W4_ERR_TIMEOUT recorded in the library's error word) and the kernel returns. No bulk
// copy, MMA or tensor memory is involved, so nothing can still be in flight when it exits.
#include "w4_sync.cuh"

namespace w4i {

namespace {

__global__ void wait_selftest_kernel(uint64_t limit_ns, int32_t *err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile int *af = &abort_flag;
    if (mbar_wait(&bar, 0u, af, err, limit_ns)) {
      // the phase cannot complete: nothing arrives on the barrier
      atomicExch(err, static_cast<int32_t>(W4_ERR_UNSUPPORTED));
    }
  }
}

}  // namespace

cudaError_t launch_wait_selftest(uint64_t limit_ns, int32_t *err, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns, err);
  return cudaGetLastError();
}

}  // namespace w4i
