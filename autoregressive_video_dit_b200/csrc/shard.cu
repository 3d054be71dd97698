// Layout steps of the head-sharded path: before the all-to-all that turns a
// sequence-sharded chunk into a head-sharded one, each rank packs its token
// slice of Q, K and V so that the heads bound for one rank are contiguous;
// after the exchange it gathers the received slices into whole-chunk
// tensors, and the reverse happens around the exchange of the output
// ("Accelerating Video Generation Inference with Sequential-Parallel 3D
// Positional Encoding Using a Global Time Index", section 2A: sequence
// parallelism with an all-to-all around attention).
//
// Each of these is a batch of row copies over a 2D index space:
// dst + i0*ds0 + i1*ds1 <- src + i0*ss0 + i1*ss1, inner bytes per row, in
// 16-byte vectors over a grid of a few waves (a warp moves whole rows).
#include "kernels.cuh"

namespace cva {

__global__ void __launch_bounds__(256) copy_rows_2d_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst,
                                                           RowCopy2D c) {
  const int64_t vec = c.inner / 16;
  const int64_t total = c.n0 * c.n1 * vec;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t v = e % vec;
    const int64_t r = e / vec;
    const int64_t i1 = r % c.n1;
    const int64_t i0 = r / c.n1;
    const uint4 x = __ldcs(reinterpret_cast<const uint4*>(src + i0 * c.ss0 + i1 * c.ss1) + v);
    reinterpret_cast<uint4*>(dst + i0 * c.ds0 + i1 * c.ds1)[v] = x;
  }
}

cudaError_t launch_copy_rows_2d(const void* src, void* dst, const RowCopy2D& c, cudaStream_t stream) {
  const int64_t total = c.n0 * c.n1 * (c.inner / 16);
  if (total == 0) return cudaSuccess;
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = (int64_t)nsm * 8;
  if (blocks > cap) blocks = cap;
  copy_rows_2d_kernel<<<(unsigned)blocks, 256, 0, stream>>>(static_cast<const uint8_t*>(src),
                                                            static_cast<uint8_t*>(dst), c);
  return cudaGetLastError();
}

}  // namespace cva
