// Self-test of the bounded device waits: one thread waits on an mbarrier that nothing ever completes,
// through the same wait routine the tensor-core kernels use, with a short budget.  The wait must give
// up, raise the timeout bit of the workspace status word and return, leaving the context usable.
#include "tc.cuh"

namespace dsa {

__global__ void __launch_bounds__(32) selftest_wait_kernel(long long budget, uint32_t *status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    tc::mbar_init(tc::smem_u32(&bar), 1);
    abort_flag = 0;
    tc::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile int *abort = &abort_flag;
    // phase 0 never completes: no thread arrives on `bar`
    if (tc::mbar_wait_for(tc::smem_u32(&bar), 0u, abort, status, budget)) set_status(status, kStatusBadIndex);
  }
}

dsa_status_t selftest_wait_launch(long long budget, void *ws, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(budget, (uint32_t *)ws);
  DSA_LAUNCH_CHECK("selftest_wait_kernel");
  return DSA_OK;
}

}  // namespace dsa
