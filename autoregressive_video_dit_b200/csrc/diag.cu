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

cudaError_t launch_exp2_poly(const float* x, float* y, int n, cudaStream_t stream) {
  const int pairs = (n + 1) / 2;
  exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, stream>>>(x, y, n);
  return cudaGetLastError();
}

}  // namespace cva
