// Diagnostic entry point: the bounded mbarrier wait of the pipeline roles,
// run on a barrier nothing arrives at, so tests can see the timeout path
// report its status without a fault or a hang.
#include "kernels.cuh"

namespace cva {

// One CTA of one warp waits, through the same bounded wait as the pipeline
// roles, on an mbarrier that nothing arrives at (no copy and no MMA is in
// flight). After `limit_ns` the wait latches CVA_DEV_TIMEOUT in the device
// error word and returns false; result[0] = 1 records that it gave up,
// result[1] = 1 that the abort flag the other roles watch was raised.
__global__ void wait_timeout_kernel(int* err, int* result, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait(&bar, 0, &abort_flag, err, limit_ns);
    result[0] = ok ? 0 : 1;
    result[1] = abort_flag;
  }
}

cudaError_t launch_wait_timeout(int* err, int* result, uint64_t limit_ns, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(err, result, limit_ns);
  return cudaGetLastError();
}

}  // namespace cva
