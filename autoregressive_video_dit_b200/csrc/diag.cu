// Diagnostic entry point: evaluates the polynomial exp2 the attention
// softmax uses for part of its exponentials, so tests can hold it to an
// error bound against the CUDA exp2f.
#include "kernels.cuh"

namespace cva {

__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = exp2_poly2(make_float2(x[i], x[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = exp2_poly2(make_float2(x[i], x[i])).x;
  }
}

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

cudaError_t launch_exp2_poly(const float* x, float* y, int n, cudaStream_t stream) {
  const int pairs = (n + 1) / 2;
  exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, stream>>>(x, y, n);
  return cudaGetLastError();
}

}  // namespace cva
