// Step 4 of the per-chunk path: two-level (frame, then block) top-k
// selection. "Light Forcing", section 2.2: for every query block a few
// history frames are picked with frame-pooled keys, then the important
// blocks inside those frames with block-pooled keys.
//
// One warp per (batch*head, query block). Scores are dot products of the
// block-pooled query with pooled keys, 32 at a time: each lane forms the
// partial dot products of its D/32 slice for 32 candidates, and a
// reduce-scatter through warp shuffles (31 exchanges) leaves candidate
// base+i's score on lane i. Every candidate becomes a 64-bit key (order-
// preserving score bits, then the complement of its position) so that a
// descending sort ranks by score and breaks ties toward the lower
// position. The warp sorts its keys with a bitonic network in its own
// slice of shared memory; the k-th key is the threshold, and the chosen
// positions are emitted in ascending order with ballots.
#include "kernels.cuh"

namespace cva {

constexpr int kSelWarps = 4;
constexpr int kSelMaxFrames = 256;

__device__ __forceinline__ uint32_t ordered_bits(float s) {
  const uint32_t u = __float_as_uint(s == 0.f ? 0.f : s);  // -0 ranks as +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ uint64_t rank_key(float s, int pos) {
  return ((uint64_t)ordered_bits(s) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)pos);
}

// Descending bitonic sort of key[0..N) (N a power of two) by one warp.
__device__ void warp_bitonic_desc(uint64_t* key, int N) {
  const int lane = threadIdx.x & 31;
  for (int k = 2; k <= N; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int p = lane; p < (N >> 1); p += 32) {
        const int i = 2 * p - (p & (j - 1));  // the member of the pair with bit j clear
        const int l = i + j;
        const uint64_t x = key[i], y = key[l];
        const bool desc = (i & k) == 0;
        if (desc ? (x < y) : (x > y)) {
          key[i] = y;
          key[l] = x;
        }
      }
      __syncwarp();
    }
  }
}

// Scores of candidates base .. base+31 (those below `count`); lane i returns
// candidate base+i's score. `row_of(c)` gives candidate c's pooled key row.
template <int D, class RowOf>
__device__ __forceinline__ float score_group(const float (&q)[D / 32], int base, int count,
                                             RowOf row_of) {
  const int lane = threadIdx.x & 31;
  float v[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    float s = 0.f;
    if (base + c < count) {
      const float* p = row_of(base + c) + lane * (D / 32);
      if constexpr (D == 128) {
        const float4 kv = *reinterpret_cast<const float4*>(p);
        s = q[0] * kv.x + q[1] * kv.y + q[2] * kv.z + q[3] * kv.w;
      } else {
        const float2 kv = *reinterpret_cast<const float2*>(p);
        s = q[0] * kv.x + q[1] * kv.y;
      }
    }
    v[c] = s;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int c = 0; c < o; ++c) {
      const float send = upper ? v[c] : v[c + o];
      const float keep = upper ? v[c + o] : v[c];
      v[c] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
    }
  }
  return v[0];
}

__host__ __device__ inline int pow2_at_least(int n) {
  int p = 32;
  while (p < n) p <<= 1;
  return p;
}

template <int D>
__global__ void __launch_bounds__(kSelWarps * 32) hsa_select_kernel(SelectArgs a, int nmax) {
  extern __shared__ uint8_t sel_smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Dims& d = a.d;
  const int u = blockIdx.x * kSelWarps + warp;
  if (u >= d.B * d.H * d.NQB) return;
  const int bh = u / d.NQB;

  // per-warp smem: keys[nmax] u64, score[nmax] f32, chosen frames[256] i32
  uint8_t* base_ptr = sel_smem + (size_t)warp * ((size_t)nmax * 12 + kSelMaxFrames * 4);
  uint64_t* key = reinterpret_cast<uint64_t*>(base_ptr);
  float* score = reinterpret_cast<float*>(base_ptr + (size_t)nmax * 8);
  int* chosen = reinterpret_cast<int*>(base_ptr + (size_t)nmax * 12);

  float q[D / 32];
  {
    const float* qp = a.qpool + (size_t)u * D + lane * (D / 32);
#pragma unroll
    for (int i = 0; i < D / 32; ++i) q[i] = qp[i];
  }
  const float* kfrm = a.kpool_frm + (size_t)bh * a.W * D;
  const float* kblk = a.kpool_blk + (size_t)bh * a.W * d.nb * D;

  // ---- level 1: frames ---------------------------------------------------
  const int F = a.F;
  const int kfe = a.k_f < F ? a.k_f : F;
  const int NF = pow2_at_least(F);
  auto frame_row = [&](int p) { return kfrm + (size_t)((a.t_lo + p) % a.W) * D; };
  for (int b0 = 0; b0 < F; b0 += 32) {
    const float s = score_group<D>(q, b0, F, frame_row);
    const int p = b0 + lane;
    if (p < F) score[p] = s;
  }
  __syncwarp();
  uint64_t thr = 1;  // every real key is above 1
  if (F > kfe) {
    for (int p = lane; p < NF; p += 32) key[p] = p < F ? rank_key(score[p], p) : 0ull;
    __syncwarp();
    warp_bitonic_desc(key, NF);
    thr = kfe > 0 ? key[kfe - 1] : ~0ull;
  }
  int nsel = 0;
  for (int b0 = 0; b0 < F; b0 += 32) {
    const int p = b0 + lane;
    const bool take = p < F && rank_key(score[p], p) >= thr;
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, take);
    if (take) chosen[nsel + __popc(bal & ((1u << lane) - 1u))] = p;
    nsel += __popc(bal);
  }
  __syncwarp();
  if (a.frame_idx) {
    for (int i = lane; i < nsel; i += 32) a.frame_idx[(size_t)u * a.k_f_stride + i] = a.t_lo + chosen[i];
  }

  // ---- level 2: blocks of the chosen frames --------------------------------
  const int C = nsel * d.nb;
  const int kb = a.k_b;
  const int NC = pow2_at_least(C);
  auto cand_row = [&](int c) {
    const int fi = c / d.nb;
    const int jj = c - fi * d.nb;
    return kblk + ((size_t)((a.t_lo + chosen[fi]) % a.W) * d.nb + jj) * D;
  };
  for (int b0 = 0; b0 < C; b0 += 32) {
    const float s = score_group<D>(q, b0, C, cand_row);
    const int c = b0 + lane;
    if (c < C) score[c] = s;
  }
  __syncwarp();
  thr = 1;
  if (C > kb) {
    for (int c = lane; c < NC; c += 32) key[c] = c < C ? rank_key(score[c], c) : 0ull;
    __syncwarp();
    warp_bitonic_desc(key, NC);
    thr = kb > 0 ? key[kb - 1] : ~0ull;
  }
  int nout = 0;
  int32_t* out = a.block_idx + (size_t)u * a.k_b_max;
  for (int b0 = 0; b0 < C; b0 += 32) {
    const int c = b0 + lane;
    const bool take = c < C && rank_key(score[c], c) >= thr;
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, take);
    if (take) {
      const int fi = c / d.nb;
      out[nout + __popc(bal & ((1u << lane) - 1u))] = (a.t_lo + chosen[fi]) * d.nb + (c - fi * d.nb);
    }
    nout += __popc(bal);
  }
  if (lane == 0 && a.block_cnt) a.block_cnt[u] = nout;
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream) {
  const int kfe = a.k_f < a.F ? a.k_f : a.F;
  const int nf = pow2_at_least(a.F);
  const int nc = pow2_at_least(kfe * a.d.nb);
  const int nmax = nf > nc ? nf : nc;
  const size_t smem = (size_t)kSelWarps * ((size_t)nmax * 12 + kSelMaxFrames * 4);
  const int units = a.d.B * a.d.H * a.d.NQB;
  dim3 grid((units + kSelWarps - 1) / kSelWarps);
  cudaError_t e;
  if (a.d.D == 128) {
    e = cudaFuncSetAttribute(hsa_select_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    hsa_select_kernel<128><<<grid, kSelWarps * 32, smem, stream>>>(a, nmax);
  } else {
    e = cudaFuncSetAttribute(hsa_select_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    hsa_select_kernel<64><<<grid, kSelWarps * 32, smem, stream>>>(a, nmax);
  }
  return cudaGetLastError();
}

}  // namespace cva
