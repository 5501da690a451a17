// Failure-detection self-test of the bounded mbarrier wait every kernel uses
// (mbar_wait, common.cuh): one thread waits for a phase of an mbarrier that
// nothing arrives on; the wait must give up after LLAMA_WAIT_LIMIT_NS of
// global-timer time, record LLAMA_DEV_TIMEOUT and return, leaving the context
// usable. No fault, trap or unbounded loop is involved.
#include "kernels.cuh"

namespace llama {

__global__ void mbarrier_selftest_kernel(int* err, unsigned long long* elapsed) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = global_timer_ns();
    (void)mbar_wait(&bar, 0, err);  // phase 0 never completes: nothing arrives on the barrier
    elapsed[0] = global_timer_ns() - t0;
  }
}

cudaError_t launch_mbarrier_selftest(int* err, unsigned long long* elapsed, cudaStream_t st) {
  mbarrier_selftest_kernel<<<1, 32, 0, st>>>(err, elapsed);
  return cudaGetLastError();
}

}  // namespace llama
