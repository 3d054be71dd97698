// Step 4 of the per-chunk path: two-level (frame, then block) top-k
// selection. "Light Forcing", section 2.2: for every query block a few
// history frames are picked with frame-pooled keys, then the important
// blocks inside those frames with block-pooled keys.
//
// One CTA of 256 threads per (batch*head, query block). Scores are dot
// products of the block-pooled query with pooled keys, 32 at a time per
// warp: each lane forms the partial dot products of its D/32 slice for 32
// candidates, and a reduce-scatter through warp shuffles (31 exchanges)
// leaves candidate base+i's score on lane i; the warps share the candidate
// groups. Every candidate becomes a 64-bit key (order-preserving score bits,
// then the complement of its position), so keys are distinct and "ranks by
// score, ties toward the lower position" is their descending order. A
// candidate's rank is the number of keys above it (each thread counts over
// the keys in shared memory); it is picked when its rank is below k. The
// picked positions are written in ascending order by a CTA-wide ordered
// compaction (warp ballots plus a scan of the per-warp counts).
//
// Top-p mode of the second level ("Sparse VideoGen2", section B, centroid
// top-p, read for key blocks): each candidate's mass is its token count times
// exp((s - s_max) / sqrt(D)); the count pass also sums the masses of the keys
// above the candidate, and the candidate is taken when that sum is below p
// times the total (the top one always, at most k_b). Masses are nonnegative
// and rounding is monotonic, so the taken set is a prefix of the ranking.
#include "kernels.cuh"

namespace cva {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelMaxFrames = 256;

__device__ __forceinline__ uint32_t ordered_bits(float s) {
  const uint32_t u = __float_as_uint(s == 0.f ? 0.f : s);  // -0 ranks as +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ uint64_t rank_key(float s, int pos) {
  return ((uint64_t)ordered_bits(s) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)pos);
}

// Scores of candidates base .. base+31 (those below `count`); lane i returns
// candidate base+i's score. Candidate c's pooled key row starts at
// rows + rowoff[c] (floats; rowoff in shared memory).
template <int D>
__device__ __forceinline__ float score_group(const float (&q)[D / 32], int base, int count,
                                             const float* rows, const int* rowoff) {
  const int lane = threadIdx.x & 31;
  float v[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    float s = 0.f;
    if (base + c < count) {
      const float* p = rows + rowoff[base + c] + lane * (D / 32);
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

// Number of keys in key[0..n) above key[i]; key[] is padded with zeros
// (below every real key) to an even length. Two keys per shared-memory
// read, the same address across the warp (a broadcast).
__device__ __forceinline__ int rank_of(const uint64_t* key, int n, int i) {
  const uint64_t x = key[i];
  const ulonglong2* k2 = reinterpret_cast<const ulonglong2*>(key);
  int r = 0;
#pragma unroll 8
  for (int j = 0; j < (n + 1) >> 1; ++j) {
    const ulonglong2 y = k2[j];
    r += (y.x > x ? 1 : 0) + (y.y > x ? 1 : 0);
  }
  return r;
}

// rank_of plus the fp32 sum of the masses m[] of the keys above key[i]
// (m[] padded like key[]).
__device__ __forceinline__ int rank_mass_of(const uint64_t* key, const float* m, int n, int i,
                                            float* above) {
  const uint64_t x = key[i];
  const ulonglong2* k2 = reinterpret_cast<const ulonglong2*>(key);
  const float2* m2 = reinterpret_cast<const float2*>(m);
  int r = 0;
  float s = 0.f;
  for (int j = 0; j < (n + 1) >> 1; ++j) {
    const ulonglong2 y = k2[j];
    const float2 w = m2[j];
    if (y.x > x) { ++r; s += w.x; }
    if (y.y > x) { ++r; s += w.y; }
  }
  *above = s;
  return r;
}

// CTA-wide max (is_max) or sum of one float per thread; all threads call it.
__device__ float cta_reduce(float v, bool is_max, float* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const float y = __shfl_xor_sync(0xFFFFFFFFu, v, o);
    v = is_max ? fmaxf(v, y) : v + y;
  }
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < kSelWarps; ++w) r = is_max ? fmaxf(r, red[w]) : r + red[w];
  __syncthreads();
  return r;
}

// Ordered compaction over positions 0..n-1: `emit(slot, pos)` for every pos
// with take(pos), slots counted in ascending pos. Returns the number taken.
// All threads of the CTA call it.
template <class Take, class Emit>
__device__ int compact(int n, int* warp_cnt, Take take, Emit emit) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int base = 0;
  for (int c0 = 0; c0 < n; c0 += kSelThreads) {
    const int c = c0 + tid;
    const bool t = c < n && take(c);
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, t);
    if (lane == 0) warp_cnt[warp] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w) {
      const int cw = warp_cnt[w];
      before += w < warp ? cw : 0;
      total += cw;
    }
    if (t) emit(base + before + __popc(bal & ((1u << lane) - 1u)), c);
    base += total;
    __syncthreads();
  }
  return base;
}

template <int D>
__global__ void __launch_bounds__(kSelThreads) hsa_select_kernel(SelectArgs a, int nmax) {
  extern __shared__ uint8_t sel_smem[];
  __shared__ int warp_cnt[kSelWarps];
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const Dims& d = a.d;
  const int u = blockIdx.x;
  const int bh = u / d.NQB;

  __shared__ float red[kSelWarps];
  // smem: keys[nmax + 1] u64, chosen frames [256] i32, row offsets [nmax] i32,
  // then (top-p) masses [nmax + 1] f32
  uint64_t* key = reinterpret_cast<uint64_t*>(sel_smem);
  int* chosen = reinterpret_cast<int*>(sel_smem + (size_t)(nmax + 1) * 8);
  int* rowoff = chosen + kSelMaxFrames;
  float* mass = reinterpret_cast<float*>(rowoff + nmax + (nmax & 1));  // 8-byte aligned

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
  for (int p = tid; p < F; p += kSelThreads) rowoff[p] = ((a.t_lo + p) % a.W) * D;
  if (tid == 0) key[F] = 0ull;  // pad to an even count
  __syncthreads();
  for (int b0 = 32 * warp; b0 < F; b0 += 32 * kSelWarps) {
    const float s = score_group<D>(q, b0, F, kfrm, rowoff);
    const int p = b0 + lane;
    if (p < F) key[p] = rank_key(s, p);
  }
  __syncthreads();
  const int nsel = compact(
      F, warp_cnt, [&](int p) { return F <= kfe || rank_of(key, F, p) < kfe; },
      [&](int slot, int p) { chosen[slot] = p; });
  if (a.frame_idx) {
    for (int i = tid; i < nsel; i += kSelThreads) a.frame_idx[(size_t)u * a.k_f_stride + i] = a.t_lo + chosen[i];
  }
  // chosen[] is complete: compact() ends with a barrier

  // ---- level 2: blocks of the chosen frames --------------------------------
  const int C = nsel * d.nb;
  const int kb = a.k_b;
  for (int c = tid; c < C; c += kSelThreads) {
    const int fi = c / d.nb;
    const int jj = c - fi * d.nb;
    rowoff[c] = (((a.t_lo + chosen[fi]) % a.W) * d.nb + jj) * D;
  }
  if (tid == 0) key[C] = 0ull;
  __syncthreads();
  const bool topp = a.topp > 0.f;
  float smax = -INFINITY;
  for (int b0 = 32 * warp; b0 < C; b0 += 32 * kSelWarps) {
    const float s = score_group<D>(q, b0, C, kblk, rowoff);
    const int c = b0 + lane;
    if (c < C) {
      key[c] = rank_key(s, c);
      if (topp) {
        mass[c] = s;
        smax = fmaxf(smax, s);
      }
    }
  }
  float thresh = 0.f;
  if (topp) {
    // masses n_c * exp((s_c - s_max) / sqrt(D)); n_c is the block's valid tokens
    smax = cta_reduce(smax, true, red);  // also orders the mass[] stores
    const float tail = (float)d.tail;
    float part = 0.f;
    for (int c = tid; c < C; c += kSelThreads) {
      const float n = (c % d.nb == d.nb - 1) ? tail : (float)d.blk;
      const float m = n * exp2f((mass[c] - smax) * a.temp_log2);
      mass[c] = m;
      part += m;
    }
    if (tid == 0) mass[C] = 0.f;
    thresh = a.topp * cta_reduce(part, false, red);
  }
  __syncthreads();
  int32_t* out = a.block_idx + (size_t)u * a.k_b_max;
  auto emit = [&](int slot, int c) {
    const int fi = c / d.nb;
    out[slot] = (a.t_lo + chosen[fi]) * d.nb + (c - fi * d.nb);
  };
  int nout;
  if (topp) {
    nout = compact(
        C, warp_cnt,
        [&](int c) {
          float above;
          const int r = rank_mass_of(key, mass, C, c, &above);
          return r < kb && (r == 0 || above < thresh);
        },
        emit);
  } else {
    nout = compact(C, warp_cnt, [&](int c) { return C <= kb || rank_of(key, C, c) < kb; }, emit);
  }
  if (tid == 0 && a.block_cnt) a.block_cnt[u] = nout;
}

// ---- pairing of 64-row query blocks into 128-row attention tiles -----------
//
// A tile of two query blocks iterates the union of their block lists, so the
// pairs are chosen by the frames the blocks picked. One CTA per
// (batch*head): its threads tabulate the number of picked frames every two
// query blocks share; then one warp walks the query blocks in order and pairs
// each unpaired one with the unpaired block after it that shares the most
// frames, ties to the lower index (one packed max-reduction per step); a
// block left over pairs with none (-1). Pair n becomes tile n.
constexpr int kPairMaxQB = 128;
constexpr int kPairWords = kSelMaxFrames / 32;
constexpr int kPairThreads = 256;

__global__ void __launch_bounds__(kPairThreads) pair_query_blocks_kernel(const int32_t* __restrict__ frame_idx,
                                                                         int kfe, int NQB, int t_lo, int MT,
                                                                         int32_t* qpair) {
  __shared__ uint32_t mask[kPairMaxQB][kPairWords];
  __shared__ uint8_t ov[kPairMaxQB][kPairMaxQB];
  const int bh = blockIdx.x;
  const int tid = threadIdx.x;
  for (int qb = tid; qb < NQB; qb += kPairThreads) {  // one thread per query block: no write races
#pragma unroll
    for (int k = 0; k < kPairWords; ++k) mask[qb][k] = 0u;
    const int32_t* fr = frame_idx + ((size_t)bh * NQB + qb) * kfe;
    for (int i = 0; i < kfe; ++i) {
      const int p = fr[i] - t_lo;  // position in the history, < 256
      if (p >= 0 && p < kSelMaxFrames) mask[qb][p >> 5] |= 1u << (p & 31);
    }
  }
  __syncthreads();
  for (int e = tid; e < NQB * NQB; e += kPairThreads) {
    const int i = e / NQB, j = e - (e / NQB) * NQB;
    int c = 0;
#pragma unroll
    for (int k = 0; k < kPairWords; ++k) c += __popc(mask[i][k] & mask[j][k]);
    ov[i][j] = (uint8_t)c;  // shared frames, at most kfe <= 255
  }
  __syncthreads();
  if (tid >= 32) return;
  const int lane = tid;
  int32_t* out = qpair + (size_t)bh * MT * 2;
  uint32_t tk[kPairMaxQB / 32] = {};  // taken query blocks, the same in every lane
  int n = 0;
  // bit i of tk, and setting it, without indexing the array at run time (registers)
  auto bit = [&](int i) {
    uint32_t w = 0u;
#pragma unroll
    for (int k = 0; k < kPairMaxQB / 32; ++k) w = (i >> 5) == k ? tk[k] : w;
    return (w >> (i & 31)) & 1u;
  };
  auto set = [&](int i) {
#pragma unroll
    for (int k = 0; k < kPairMaxQB / 32; ++k)
      if ((i >> 5) == k) tk[k] |= 1u << (i & 31);
  };
  for (int i = 0; i < NQB; ++i) {
    if (bit(i)) continue;
    // key: shared frames + 1, then the complement of j (ties to the lower j); 0: none
    unsigned key = 0u;
#pragma unroll
    for (int k = 0; k < kPairMaxQB / 32; ++k) {
      const int j = 32 * k + lane;
      if (j > i && j < NQB && !((tk[k] >> lane) & 1u)) key = max(key, (1u + ov[i][j]) << 16 | (0xFFFFu - (unsigned)j));
    }
    key = __reduce_max_sync(0xFFFFFFFFu, key);
    const int best = key ? (int)(0xFFFFu - (key & 0xFFFFu)) : -1;
    set(i);
    if (best >= 0) set(best);
    if (lane == 0) {
      out[2 * n] = i;
      out[2 * n + 1] = best;
    }
    ++n;
  }
  for (int t = n + lane; t < MT; t += 32) {  // tiles without query blocks (none when MT = ceil(NQB / 2))
    out[2 * t] = -1;
    out[2 * t + 1] = -1;
  }
}

cudaError_t launch_pair_query_blocks(const int32_t* frame_idx, int kfe, const Dims& d, int t_lo, int F, int MT,
                                     int32_t* qpair, cudaStream_t stream) {
  if (d.NQB > kPairMaxQB || F > kSelMaxFrames || kfe < 1 || kfe > 255) return cudaErrorInvalidValue;
  pair_query_blocks_kernel<<<d.B * d.H, kPairThreads, 0, stream>>>(frame_idx, kfe, d.NQB, t_lo, MT, qpair);
  return cudaGetLastError();
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream) {
  const int kfe = a.k_f < a.F ? a.k_f : a.F;
  const int nmax = a.F > kfe * a.d.nb ? a.F : kfe * a.d.nb;
  const size_t smem = (size_t)(nmax + 1) * 8 + kSelMaxFrames * 4 + (size_t)nmax * 4 +
                      (a.topp > 0.f ? (size_t)(nmax + 2) * 4 : 0);
  const int units = a.d.B * a.d.H * a.d.NQB;
  dim3 grid(units);
  cudaError_t e;
  if (a.d.D == 128) {
    e = cudaFuncSetAttribute(hsa_select_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    hsa_select_kernel<128><<<grid, kSelThreads, smem, stream>>>(a, nmax);
  } else {
    e = cudaFuncSetAttribute(hsa_select_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    hsa_select_kernel<64><<<grid, kSelThreads, smem, stream>>>(a, nmax);
  }
  return cudaGetLastError();
}

}  // namespace cva
