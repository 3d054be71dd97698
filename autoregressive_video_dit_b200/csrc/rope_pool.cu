// Steps 1-3 of the per-chunk path: Causal-RoPE with a global time index,
// the frame-cache append, and block/frame mean pooling.
//
// "Accelerating Video Generation Inference with Sequential-Parallel 3D
// Positional Encoding Using a Global Time Index", section 2B: a token of
// local frame f in a chunk that starts at global frame t0 is rotated with
// temporal coordinate t0 + f; section 2C: cos/sin come from precomputed
// contiguous tables. "Light Forcing", section 2.2 (token compression):
// queries and keys are mean-pooled per block and per frame.
//
// One CTA handles one (batch*head, frame, block) tile of up to three
// tensors (Q, K, V) in a single pass over HBM: each thread owns 8
// consecutive elements (one 16-byte vector) of a row, so a warp reads and
// writes whole 256-byte rows. Block sums are reduced in a fixed order
// (deterministic), from the bf16 values actually stored.
#include "kernels.cuh"

namespace cva {

template <int D>
__global__ void __launch_bounds__(256) rope_pool_kernel(RopePoolArgs a) {
  constexpr int kCG = D / 8;          // column groups (16-byte vectors) per row
  constexpr int kRP = 256 / kCG;      // rows per pass
  __shared__ float red[kRP][D];

  const Dims& d = a.d;
  const int f = blockIdx.x / d.nb;
  const int j = blockIdx.x - f * d.nb;
  const int bh = blockIdx.y;
  const int b = bh / d.H;
  const int h = bh - b * d.H;
  const int tid = threadIdx.x;
  const int cg = tid % kCG;
  const int rg = tid / kCG;
  const int valid = (j == d.nb - 1) ? d.tail : d.blk;
  const int t = a.t0 + f;
  const int slot = t % a.W;

  // Rotary table lookups of this thread's 4 pairs: axis and local index.
  const float* ctab[4];
  const float* stab[4];
  int axis[4];
  int pstride[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int p = cg * 4 + i;
    if (p < a.tab.pt) {
      axis[i] = 0; ctab[i] = a.tab.cos_t + p; stab[i] = a.tab.sin_t + p; pstride[i] = a.tab.pt;
    } else if (p < a.tab.pt + a.tab.ph) {
      const int q = p - a.tab.pt;
      axis[i] = 1; ctab[i] = a.tab.cos_h + q; stab[i] = a.tab.sin_h + q; pstride[i] = a.tab.ph;
    } else {
      const int q = p - a.tab.pt - a.tab.ph;
      axis[i] = 2; ctab[i] = a.tab.cos_w + q; stab[i] = a.tab.sin_w + q; pstride[i] = a.tab.pw;
    }
  }

  for (int jb = 0; jb < a.njobs; ++jb) {
    const StreamJob job = a.job[jb];
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;

    for (int r = rg; r < d.blk; r += kRP) {
      const int rr = j * d.blk + r;            // row inside the frame (padded)
      uint4 y = make_uint4(0u, 0u, 0u, 0u);
      if (r < valid) {
        size_t src_off;
        if (job.src_layout == kTokenMajor) {
          const size_t n = (size_t)f * d.T_f + rr;
          src_off = (((size_t)b * d.Lq + n) * d.H + h) * D;
        } else {
          src_off = ((size_t)bh * d.Fc * d.T_pad + (size_t)f * d.T_pad + rr) * D;
        }
        const uint4 x = *reinterpret_cast<const uint4*>(job.src + src_off + cg * 8);
        if (job.rotate) {
          const int hh = rr / d.Fw;
          const int ww = rr - hh * d.Fw;
          const uint32_t xin[4] = {x.x, x.y, x.z, x.w};
          uint32_t yout[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int pos = axis[i] == 0 ? t : (axis[i] == 1 ? hh : ww);
            const float c = __ldg(ctab[i] + (size_t)pos * pstride[i]);
            const float s = __ldg(stab[i] + (size_t)pos * pstride[i]);
            const float x0 = bf16_lo(xin[i]);
            const float x1 = bf16_hi(xin[i]);
            yout[i] = pack_bf16(x0 * c - x1 * s, x0 * s + x1 * c);
          }
          y = make_uint4(yout[0], yout[1], yout[2], yout[3]);
        } else {
          y = x;
        }
        if (job.pool) {
          acc[0] += bf16_lo(y.x); acc[1] += bf16_hi(y.x);
          acc[2] += bf16_lo(y.y); acc[3] += bf16_hi(y.y);
          acc[4] += bf16_lo(y.z); acc[5] += bf16_hi(y.z);
          acc[6] += bf16_lo(y.w); acc[7] += bf16_hi(y.w);
        }
      }
      if (job.dst) {
        if (job.dst_layout == kTokenMajor) {
          if (r < valid) {
            const size_t n = (size_t)f * d.T_f + rr;
            *reinterpret_cast<uint4*>(job.dst + (((size_t)b * d.Lq + n) * d.H + h) * D + cg * 8) = y;
          }
        } else if (job.dst_layout == kHeadMajor) {
          *reinterpret_cast<uint4*>(
              job.dst + ((size_t)bh * d.Fc * d.T_pad + (size_t)f * d.T_pad + rr) * D + cg * 8) = y;
        } else {
          *reinterpret_cast<uint4*>(
              job.dst + (((size_t)bh * a.W + slot) * d.T_pad + rr) * D + cg * 8) = y;
        }
      }
    }

    if (job.pool) {
#pragma unroll
      for (int i = 0; i < 8; ++i) red[rg][cg * 8 + i] = acc[i];
      __syncthreads();
      if (tid < D) {
        float s = 0.f;
#pragma unroll 4
        for (int g = 0; g < kRP; ++g) s += red[g][tid];
        const float mean = s / (float)valid;
        size_t off;
        if (job.pool_layout == kPoolChunk) {
          off = ((size_t)bh * d.NQB + (size_t)f * d.nb + j) * D + tid;
        } else {
          off = (((size_t)bh * a.W + slot) * d.nb + j) * D + tid;
        }
        job.pool[off] = mean;
      }
      __syncthreads();
    }
  }
}

// Frame means from block means: sum_j count_j * mean_j / T_f, in block order.
__global__ void frame_pool_kernel(FramePoolArgs a) {
  const Dims& d = a.d;
  const int f = blockIdx.x;
  const int bh = blockIdx.y;
  const int c = threadIdx.x;
  if (c >= d.D) return;
  const float* src;
  float* dst;
  if (a.layout == kPoolChunk) {
    src = a.blk_pool + ((size_t)bh * d.NQB + (size_t)f * d.nb) * d.D;
    dst = a.frm_pool + ((size_t)bh * d.Fc + f) * d.D;
  } else {
    const int slot = (a.t0 + f) % a.W;
    src = a.blk_pool + ((size_t)bh * a.W + slot) * d.nb * d.D;
    dst = a.frm_pool + ((size_t)bh * a.W + slot) * d.D;
  }
  float s = 0.f;
  for (int j = 0; j < d.nb; ++j) {
    const float cnt = (float)((j == d.nb - 1) ? d.tail : d.blk);
    s += cnt * src[(size_t)j * d.D + c];
  }
  dst[c] = s / (float)d.T_f;
}

// ---- host-side launchers (called from api.cu) -----------------------------

cudaError_t launch_rope_pool(const RopePoolArgs& a, cudaStream_t stream) {
  dim3 grid(a.d.Fc * a.d.nb, a.d.B * a.d.H);
  if (a.d.D == 128) {
    rope_pool_kernel<128><<<grid, 256, 0, stream>>>(a);
  } else {
    rope_pool_kernel<64><<<grid, 256, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_frame_pool(const FramePoolArgs& a, cudaStream_t stream) {
  dim3 grid(a.d.Fc, a.d.B * a.d.H);
  frame_pool_kernel<<<grid, a.d.D, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace cva
