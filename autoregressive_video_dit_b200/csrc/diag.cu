// Diagnostic entry points: the bounded mbarrier wait of the pipeline roles,
// run on a barrier nothing arrives at, so tests can see the timeout path
// report its status without a fault or a hang; and the tensor-core time of
// one tcgen05.mma shape, which decides how attention tiles are laid out.
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

// One CTA per SM: one thread issues `iters` x 4 back-to-back
// tcgen05.mma kind::f16 (bf16 operands of zeros in shared memory, fp32
// accumulator in tensor memory) of shape M x N x 16, commits, and waits
// (bounded) for completion; cycles[blockIdx.x] = clock64 span.
__global__ void __launch_bounds__(128, 1) mma_cycles_kernel(int M, int N, int iters,
                                                             unsigned long long* cycles, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t tslot;
  uint8_t* A = smem;          // up to 128 rows x 128 B, 128-byte swizzle
  uint8_t* B = smem + 16384;  // up to 256 rows x 128 B
  for (int i = threadIdx.x; i < (16384 + 32768) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  fence_proxy_async_smem();
  if (threadIdx.x < 32) {
    tmem_alloc(&tslot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  if (threadIdx.x == 0) {
    const uint32_t idesc = idesc_bf16_f32(M, N, 0, 0);
    const uint64_t ad = smem_desc_sw128(smem_u32(A), 16, 1024);
    const uint64_t bd = smem_desc_sw128(smem_u32(B), 16, 1024);
    const unsigned long long t0 = clock64();
    for (int i = 0; i < iters; ++i) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_ss(tmem, ad + (uint64_t)((k * 32) >> 4), bd + (uint64_t)((k * 32) >> 4), idesc, (i | k) ? 1u : 0u);
    }
    mma_commit(&bar);
    const uint64_t g0 = globaltimer_ns();
    bool done = true;
    while (!mbar_try_wait(&bar, 0)) {
      if (globaltimer_ns() - g0 > kWaitLimitNs) {
        done = false;
        break;
      }
    }
    const unsigned long long t1 = clock64();
    if (!done) latch_error(err, CVA_DEV_TIMEOUT);
    cycles[blockIdx.x] = t1 - t0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x < 32) tmem_dealloc(tmem, 512);
}

cudaError_t launch_mma_cycles(int M, int N, int iters, unsigned long long* cycles, int sms, int* err,
                              cudaStream_t stream) {
  const int smem = 16384 + 32768 + 1024;
  cudaError_t e = cudaFuncSetAttribute(mma_cycles_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  mma_cycles_kernel<<<sms, 128, smem, stream>>>(M, N, iters, cycles, err);
  return cudaGetLastError();
}

}  // namespace cva
