// Step 4 of the per-chunk path: two-level (frame, then block) top-k
// selection. "Light Forcing", section 2.2: for every query block a few
// history frames are picked with frame-pooled keys, then the important
// blocks inside those frames with block-pooled keys.
//
// P warps per (batch*head, query block) -- four, two or one, as many as
// keep every query block of the call resident at once -- and 16 / P query
// blocks of a head to a CTA (so that they share the pooled keys in L1),
// with no barrier wider than a query block's warps: the work of a query block is a
// chain of dependent steps (load, score, pick, load, score, pick), so its
// latency is what counts. Scores are dot products of the block-pooled
// query with pooled keys, 32 at a time per warp: each lane forms the
// partial dot products of its D/32 slice for 32 candidates, and a
// reduce-scatter through warp shuffles (31 exchanges) leaves candidate
// base+i's score on lane i; the query block's warps share the candidate
// groups of the second level. Every candidate becomes a 64-bit key (order-preserving
// score bits, then the complement of its position), so keys are distinct
// and "ranks by score, ties toward the lower position" is their descending
// order. The k-th largest key is found by a radix select over the key
// digits in a histogram private to the query block, and the candidates
// whose keys are at least that large are written in ascending position by
// ballot compaction. Before it scores the frames, the query block asks L2
// to fetch its share of the head's block-pooled keys, which the second
// level reads after the frame pick.
//
// Top-p mode of the second level ("Sparse VideoGen2", section B, centroid
// top-p, read for key blocks): each candidate's mass is its token count times
// exp((s - s_max) / sqrt(D)); a count over the keys also sums the masses of
// the keys above each candidate, and the candidate is taken when that sum is
// below p times the total (the top one always, at most k_b). Masses are
// nonnegative and rounding is monotonic, so the taken set is a prefix of the
// ranking.
#include "kernels.cuh"

namespace cva {

constexpr int kSelThreads = 512;             // 16 warps: 16 / P query blocks of P warps
constexpr int kSelSmSlots = 32;              // warps per SM at the kernel's 64 registers
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

// The smallest of the k largest keys of key[0..n) (keys distinct, 1 <= k
// <= n), so that exactly the k largest satisfy key >= result; called by
// the whole warp. Radix select, most significant 8-bit digit first: a pass
// counts the keys that match the digits fixed so far into 256 bins, and
// the lanes (eight bins each) find by a scan the bin where the count from
// the top reaches the number still needed; when that bin holds exactly
// that many keys (at the last digit always, the keys being distinct) all
// of them are taken and the threshold is known. `hist`: 256 ints of
// shared memory private to the warp.
__device__ uint64_t warp_kth_largest(const uint64_t* key, int n, int k, int* hist) {
  const int lane = threadIdx.x & 31;
  uint64_t prefix = 0ull;
  int need = k;
  for (int shift = 56;; shift -= 8) {
#pragma unroll
    for (int i = 0; i < 8; ++i) hist[32 * i + lane] = 0;
    __syncwarp();
    for (int c = lane; c < n; c += 32) {
      const uint64_t x = key[c];
      if (shift == 56 || (x >> (shift + 8)) == (prefix >> (shift + 8)))
        atomicAdd(&hist[(int)((x >> shift) & 255u)], 1);
    }
    __syncwarp();
    int v[8], sum = 0;  // lane l: bins 255 - 8l down to 248 - 8l
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      v[j] = hist[255 - 8 * lane - j];
      sum += v[j];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += t;
    }
    const int excl = incl - sum;
    int digit = 0, above = excl, cnt = 0;
    const bool mine = excl < need && need <= incl;   // exactly one lane
    if (mine) {
      int j = 0;
      while (above + v[j] < need) above += v[j++];
      digit = 255 - 8 * lane - j;
      cnt = v[j];
    }
    const int src = __ffs(__ballot_sync(0xFFFFFFFFu, mine)) - 1;
    digit = __shfl_sync(0xFFFFFFFFu, digit, src);
    above = __shfl_sync(0xFFFFFFFFu, above, src);
    cnt = __shfl_sync(0xFFFFFFFFu, cnt, src);
    prefix |= (uint64_t)digit << shift;
    need -= above;
    if (cnt == need || shift == 0) return prefix;
    __syncwarp();
  }
}

// Number of keys in key[0..n) above key[i], and the fp32 sum of the masses
// m[] of those keys; key[] and m[] are padded with a zero to an even
// length (below every real key, no mass). Two keys per shared-memory read.
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

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Ordered compaction over positions 0..n-1 by one warp: `emit(slot, pos)`
// for every pos with take(pos), slots counted in ascending pos. Returns the
// number taken.
template <class Take, class Emit>
__device__ __forceinline__ int warp_compact(int n, Take take, Emit emit) {
  const int lane = threadIdx.x & 31;
  int base = 0;
  for (int c0 = 0; c0 < n; c0 += 32) {
    const int c = c0 + lane;
    const bool t = c < n && take(c);
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, t);
    if (t) emit(base + __popc(bal & ((1u << lane) - 1u)), c);
    base += __popc(bal);
  }
  return base;
}

// Shared memory of one query block for at most nmax candidates: keys
// (nmax + 2), row offsets or top-p take flags (nmax, rounded up to even so
// that the masses stay 8-byte aligned), histogram (256), chosen frames,
// the group's partial max / sum (2 x 4), masses (nmax + 2, top-p).
inline size_t sel_group_bytes(int nmax, bool topp) {
  const size_t b = (size_t)(nmax + 2) * 8 + (size_t)(nmax + (nmax & 1)) * 4 + 256 * 4 +
                   kSelMaxFrames * 4 + 8 * 4 + (topp ? (size_t)(nmax + 2) * 4 : 0);
  return (b + 15) & ~size_t(15);
}

template <int D, int P>
__global__ void __launch_bounds__(kSelThreads, 2) hsa_select_kernel(SelectArgs a, int nmax, int units,
                                                                      int group_bytes) {
  extern __shared__ __align__(16) uint8_t sel_smem[];
  constexpr int kQbs = kSelThreads / (32 * P);  // query blocks per CTA
  constexpr int kGT = 32 * P;                   // threads per query block
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = warp / P;       // query block of the CTA
  const int wq = warp - g * P;  // warp within it
  const int gt = 32 * wq + lane;
  const Dims& d = a.d;
  griddep_launch_dependents();
  const int u = blockIdx.x * kQbs + g;
  if (u >= units) return;  // the query block's warps together
  // barrier over the query block's warps: the warp itself, or named barrier
  // 1 + g (immediate ids, so that the kernel holds only the ids it uses)
  auto gsync = [g] {
    static_assert(P == 1 || P == 2 || P == 4, "warps per query block");
    if constexpr (P == 1) {
      __syncwarp();
    } else {
      switch (g) {
        case 0: asm volatile("bar.sync 1, %0;" ::"n"(kGT) : "memory"); break;
        case 1: asm volatile("bar.sync 2, %0;" ::"n"(kGT) : "memory"); break;
        case 2: asm volatile("bar.sync 3, %0;" ::"n"(kGT) : "memory"); break;
        case 3: asm volatile("bar.sync 4, %0;" ::"n"(kGT) : "memory"); break;
        case 4: asm volatile("bar.sync 5, %0;" ::"n"(kGT) : "memory"); break;
        case 5: asm volatile("bar.sync 6, %0;" ::"n"(kGT) : "memory"); break;
        case 6: asm volatile("bar.sync 7, %0;" ::"n"(kGT) : "memory"); break;
        default: asm volatile("bar.sync 8, %0;" ::"n"(kGT) : "memory"); break;
      }
    }
  };
  const int bh = u / d.NQB;
  const bool topp = a.topp > 0.f;
  uint8_t* base = sel_smem + (size_t)g * group_bytes;
  uint64_t* key = reinterpret_cast<uint64_t*>(base);
  int* rowoff = reinterpret_cast<int*>(key + nmax + 2);
  int* hist = rowoff + nmax + (nmax & 1);
  int* chosen = hist + 256;
  float* red = reinterpret_cast<float*>(chosen + kSelMaxFrames);
  float* mass = red + 8;

  const float* kfrm = a.kpool_frm + (size_t)bh * a.W * D;
  const float* kblk = a.kpool_blk + (size_t)bh * a.W * d.nb * D;
  const int F = a.F;
  {
    // L2 prefetch of this query block's share of the head's history frame
    // and block means (128-byte lines; the head's query blocks take every
    // NQB-th line). No kernel of the call writes them, so this may run
    // before the wait for the preceding launch.
    const int r = u - bh * d.NQB;
    const int lpf = d.nb * D / 32;  // block-mean lines per frame
    constexpr int kFrmLines = D / 32;
    for (int l = r + d.NQB * gt; l < F * (lpf + kFrmLines); l += kGT * d.NQB) {
      const float* line;
      if (l < F * lpf) {
        const int p = l / lpf;
        line = kblk + (size_t)((a.t_lo + p) % a.W) * d.nb * D + (size_t)(l - p * lpf) * 32;
      } else {
        const int lf = l - F * lpf;
        const int p = lf / kFrmLines;
        line = kfrm + (size_t)((a.t_lo + p) % a.W) * D + (size_t)(lf - p * kFrmLines) * 32;
      }
      asm volatile("prefetch.global.L2 [%0];" ::"l"(line));
    }
  }
  griddep_wait();  // the pooled queries come from the preceding rotation
  float q[D / 32];
  {
    const float* qp = a.qpool + (size_t)u * D + lane * (D / 32);
#pragma unroll
    for (int i = 0; i < D / 32; ++i) q[i] = qp[i];
  }

  // ---- level 1: frames (warp 0 of the query block) --------------------------
  const int kfe = a.k_f < F ? a.k_f : F;  // frames picked: all, or exactly k_f
  if (wq == 0) {
    for (int p = lane; p < F; p += 32) rowoff[p] = ((a.t_lo + p) % a.W) * D;
    __syncwarp();
    for (int b0 = 0; b0 < F; b0 += 32) {
      const float s = score_group<D>(q, b0, F, kfrm, rowoff);
      const int p = b0 + lane;
      if (p < F) key[p] = rank_key(s, p);
    }
    __syncwarp();
    if (F <= kfe) {
      for (int p = lane; p < F; p += 32) chosen[p] = p;
    } else {
      const uint64_t kth = warp_kth_largest(key, F, kfe, hist);
      warp_compact(F, [&](int p) { return key[p] >= kth; }, [&](int slot, int p) { chosen[slot] = p; });
    }
    __syncwarp();
    if (a.frame_idx) {
      for (int i = lane; i < kfe; i += 32) a.frame_idx[(size_t)u * a.k_f_stride + i] = a.t_lo + chosen[i];
    }
  }
  gsync();

  // ---- level 2: blocks of the chosen frames (all the query block's warps) ----
  const int C = kfe * d.nb;
  const int kb = a.k_b;
  for (int c = gt; c < C; c += kGT) {
    const int fi = c / d.nb;
    const int jj = c - fi * d.nb;
    rowoff[c] = (((a.t_lo + chosen[fi]) % a.W) * d.nb + jj) * D;
  }
  if (gt == 0) {
    key[C] = 0ull;  // pad to an even count
    if (topp) mass[C] = 0.f;
  }
  gsync();
  float smax = -INFINITY;
  for (int b0 = 32 * wq; b0 < C; b0 += kGT) {
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
    smax = warp_max(smax);
    if (lane == 0) red[wq] = smax;
    gsync();
    smax = red[0];
#pragma unroll
    for (int w = 1; w < P; ++w) smax = fmaxf(smax, red[w]);
    const float tail = (float)d.tail;
    float part = 0.f;
    for (int c = gt; c < C; c += kGT) {
      const float n = (c % d.nb == d.nb - 1) ? tail : (float)d.blk;
      const float m = n * exp2f((mass[c] - smax) * a.temp_log2);
      mass[c] = m;
      part += m;
    }
    part = warp_sum(part);
    if (lane == 0) red[4 + wq] = part;
    gsync();
    float total = red[4];
#pragma unroll
    for (int w = 1; w < P; ++w) total += red[4 + w];
    thresh = a.topp * total;
    // take flags over the row offsets, which the scoring no longer needs
    for (int c = gt; c < C; c += kGT) {
      float above;
      const int r = rank_mass_of(key, mass, C, c, &above);
      rowoff[c] = (r < kb && (r == 0 || above < thresh)) ? 1 : 0;
    }
  }
  gsync();
  if (wq != 0) return;
  int32_t* out = a.block_idx + (size_t)u * a.k_b_max;
  auto emit = [&](int slot, int c) {
    const int fi = c / d.nb;
    out[slot] = (a.t_lo + chosen[fi]) * d.nb + (c - fi * d.nb);
  };
  int nout;
  if (topp) {
    nout = warp_compact(C, [&](int c) { return rowoff[c] != 0; }, emit);
  } else if (C <= kb || kb <= 0) {
    nout = warp_compact(C, [&](int) { return kb > 0; }, emit);
  } else {
    const uint64_t kth = warp_kth_largest(key, C, kb, hist);
    nout = warp_compact(C, [&](int c) { return key[c] >= kth; }, emit);
  }
  if (lane == 0 && a.block_cnt) a.block_cnt[u] = nout;
}

// ---- pairing of 64-row query blocks into 128-row attention tiles -----------
//
// A tile of two query blocks iterates the union of their block lists, so the
// pairs are chosen by the frames the blocks picked. One CTA per
// (batch*head), in rounds: every unpaired block names its best unpaired
// partner -- the one sharing the most picked frames, ties to the lower
// index -- and blocks that name each other pair up. The best remaining pair
// overall (most shared frames, then lowest indices) always names itself
// both ways, so every round pairs at least two blocks; when one block is
// left it pairs with none (-1). Overlaps of kPairLevels - 1 frames or more
// count as equal. Tile n holds the pair whose lower block is the n-th
// lowest. To make a round cheap, the CTA first tabulates, for every block i
// and overlap v, the set of blocks j != i sharing exactly v frames with i
// as a 128-bit mask, and which overlaps occur: a block's best partner is
// then the lowest unpaired block in the highest overlap that still has one
// (a few bit operations, usually on the first mask it reads).
constexpr int kPairMaxQB = 128;
constexpr int kPairWords = kSelMaxFrames / 32;
constexpr int kPairThreads = 1024;  // threads 0..127: one per query block; all: the level masks
constexpr int kPairLevels = 32;

__global__ void __launch_bounds__(kPairThreads) pair_query_blocks_kernel(const int32_t* __restrict__ frame_idx,
                                                                         int kfe, int NQB, int t_lo, int F,
                                                                         int MT, int32_t* qpair) {
  __shared__ uint32_t mask[kPairWords][kPairMaxQB];  // word-major: lanes read consecutive words
  __shared__ uint32_t occurs[kPairMaxQB];            // bit v: some j shares v frames with i
  __shared__ int best[kPairMaxQB];
  __shared__ int partner[kPairMaxQB];                // -2: unpaired so far
  __shared__ uint32_t freew[kPairMaxQB / 32];       // unpaired blocks, one word per warp
  __shared__ int wcnt[kPairMaxQB / 32];
  extern __shared__ uint32_t lvl[];                  // [NQB][L][4]
  const int L = kfe + 1 < kPairLevels ? kfe + 1 : kPairLevels;
  const int nw = (F + 31) >> 5;
  const int bh = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i = tid;  // the block this thread speaks for
  griddep_launch_dependents();
  griddep_wait();  // the frame lists come from the preceding selection
  if (i < NQB) {
    uint32_t m[kPairWords] = {};
    const int32_t* fr = frame_idx + ((size_t)bh * NQB + i) * kfe;
#pragma unroll 4
    for (int k = 0; k < kfe; ++k) {
      const int p = fr[k] - t_lo;  // position in the history, < 256
#pragma unroll
      for (int w = 0; w < kPairWords; ++w)
        if (p >= 32 * w && p < 32 * w + 32) m[w] |= 1u << (p & 31);
    }
#pragma unroll
    for (int w = 0; w < kPairWords; ++w) mask[w][i] = m[w];
    partner[i] = -2;
    occurs[i] = 0u;
  }
  __syncthreads();
  // Level masks, one (block r, 32 blocks j) item per warp step: the lanes
  // ballot the five bits of their overlaps, and lane v assembles the word of
  // overlap v from them (bit-sliced equality); a word's lane also records
  // whether the overlap occurs. Each item is a short dependent chain, so the
  // items are spread over all 32 warps.
  for (int r = warp; r < NQB; r += kPairThreads / 32) {
    // the four 32-block groups as independent chains
    int ov[4];
    bool valid[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int j = 32 * k + lane;
      valid[k] = j < NQB && j != r;
      int o = 0;
      if (valid[k]) {
        for (int w = 0; w < nw; ++w) o += __popc(mask[w][r] & mask[w][j]);
        o = o < L - 1 ? o : L - 1;
      }
      ov[k] = o;
    }
    uint32_t word[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) word[k] = __ballot_sync(0xFFFFFFFFu, valid[k]);
#pragma unroll
    for (int bit = 0; bit < 5; ++bit) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t bb = __ballot_sync(0xFFFFFFFFu, (ov[k] >> bit) & 1);
        word[k] &= ((lane >> bit) & 1) ? bb : ~bb;
      }
    }
    if (lane < L) {
      uint4 wv = make_uint4(word[0], word[1], word[2], word[3]);
      reinterpret_cast<uint4*>(lvl)[r * L + lane] = wv;
    }
    const uint32_t occ = __ballot_sync(0xFFFFFFFFu, lane < L && (word[0] | word[1] | word[2] | word[3]) != 0u);
    if (lane == 0) occurs[r] = occ;
  }
  if (tid < kPairMaxQB && lane == 0) {
    const int lo = 32 * warp;
    freew[warp] = NQB >= lo + 32 ? 0xFFFFFFFFu : (NQB > lo ? (1u << (NQB - lo)) - 1u : 0u);
  }
  __syncthreads();
  // The rounds involve one thread per query block: warps 0-3, with their
  // own named barrier; the other warps are done.
  if (tid >= kPairMaxQB) return;
  auto qsync = [] { asm volatile("bar.sync 1, %0;" ::"n"(kPairMaxQB) : "memory"); };
  int nfree = NQB;
  // every round pairs at least two blocks, so NQB / 2 rounds suffice
  for (int round = 0; nfree >= 2 && round < kPairMaxQB / 2; ++round) {
    const uint32_t f0 = freew[0], f1 = freew[1], f2 = freew[2], f3 = freew[3];
    const uint32_t mine = warp == 0 ? f0 : (warp == 1 ? f1 : (warp == 2 ? f2 : f3));
    if ((mine >> lane) & 1u) {
      int b = -1;
      uint32_t occ = occurs[i];
      while (occ) {
        const int v = 31 - __clz(occ);
        occ &= ~(1u << v);
        const uint4 c = reinterpret_cast<const uint4*>(lvl)[i * L + v];
        const uint32_t c0 = c.x & f0, c1 = c.y & f1, c2 = c.z & f2, c3 = c.w & f3;
        if (c0 | c1 | c2 | c3) {
          b = c0 ? __ffs(c0) - 1 : (c1 ? 31 + __ffs(c1) : (c2 ? 63 + __ffs(c2) : 95 + __ffs(c3)));
          break;
        }
      }
      best[i] = b;
    }
    qsync();
    // pair the blocks that name each other; each pair is written by its lower block
    if ((mine >> lane) & 1u) {
      const int b = best[i];
      if (b > i && best[b] == i) {
        partner[i] = b;
        partner[b] = i;
      }
    }
    qsync();
    const uint32_t still = __ballot_sync(0xFFFFFFFFu, ((mine >> lane) & 1u) && partner[i] < 0);
    if (lane == 0) {
      freew[warp] = still;
      wcnt[warp] = __popc(still);
    }
    qsync();
    nfree = wcnt[0] + wcnt[1] + wcnt[2] + wcnt[3];
  }
  // tile n: the pair (or the lone block) whose lower block is the n-th lowest
  const bool lead = i < NQB && (partner[i] > i || partner[i] == -2);
  const uint32_t bal = __ballot_sync(0xFFFFFFFFu, lead);
  qsync();  // every thread has read wcnt
  if (lane == 0) wcnt[warp] = __popc(bal);
  qsync();
  int before = __popc(bal & ((1u << lane) - 1u));
  for (int w = 0; w < warp; ++w) before += wcnt[w];
  const int n = wcnt[0] + wcnt[1] + wcnt[2] + wcnt[3];
  int32_t* out = qpair + (size_t)bh * MT * 2;
  if (lead && before < MT) {
    out[2 * before] = i;
    out[2 * before + 1] = partner[i] >= 0 ? partner[i] : -1;
  }
  for (int t = n + tid; t < MT; t += kPairMaxQB) {  // tiles without query blocks (none when MT = ceil(NQB / 2))
    out[2 * t] = -1;
    out[2 * t + 1] = -1;
  }
}

cudaError_t launch_pair_query_blocks(const int32_t* frame_idx, int kfe, const Dims& d, int t_lo, int F, int MT,
                                     int32_t* qpair, cudaStream_t stream, bool dependent) {
  if (d.NQB > kPairMaxQB || F > kSelMaxFrames || kfe < 1 || kfe > 255) return cudaErrorInvalidValue;
  const int L = kfe + 1 < kPairLevels ? kfe + 1 : kPairLevels;
  const size_t smem = (size_t)d.NQB * L * 16;
  cudaError_t e = cudaFuncSetAttribute(pair_query_blocks_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  return launch_kernel(pair_query_blocks_kernel, dim3(d.B * d.H), dim3(kPairThreads), smem, stream, dependent,
                       frame_idx, kfe, d.NQB, t_lo, F, MT, qpair);
}

template <int D, int P>
static cudaError_t launch_select_p(const SelectArgs& a, int nmax, int units, size_t gb, cudaStream_t stream,
                                   bool dependent) {
  constexpr int qbs = kSelThreads / (32 * P);
  const size_t smem = gb * qbs;
  cudaError_t e = cudaFuncSetAttribute(hsa_select_kernel<D, P>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  return launch_kernel(hsa_select_kernel<D, P>, dim3((units + qbs - 1) / qbs), dim3(kSelThreads), smem, stream,
                       dependent, a, nmax, units, (int)gb);
}

// Warps per query block: as many as keep every query block resident at
// once (the work of one is a latency chain that more warps shorten), and
// as shared memory allows.
cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream, bool dependent) {
  const int kfe = a.k_f < a.F ? a.k_f : a.F;
  const int nmax = a.F > kfe * a.d.nb ? a.F : kfe * a.d.nb;
  const size_t gb = sel_group_bytes(nmax, a.topp > 0.f);
  const int units = a.d.B * a.d.H * a.d.NQB;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const size_t smem_cap = 100 * 1024;  // two CTAs per SM
  int P = 4;
  while (P > 1 && (int64_t)sms * kSelSmSlots / P < units) P >>= 1;
  while (P < 4 && gb * (kSelThreads / (32 * P)) > smem_cap) P <<= 1;
  if (gb * (kSelThreads / (32 * P)) > smem_cap * 2) return cudaErrorInvalidValue;
  if (a.d.D == 128) {
    if (P == 4) return launch_select_p<128, 4>(a, nmax, units, gb, stream, dependent);
    if (P == 2) return launch_select_p<128, 2>(a, nmax, units, gb, stream, dependent);
    return launch_select_p<128, 1>(a, nmax, units, gb, stream, dependent);
  }
  if (P == 4) return launch_select_p<64, 4>(a, nmax, units, gb, stream, dependent);
  if (P == 2) return launch_select_p<64, 2>(a, nmax, units, gb, stream, dependent);
  return launch_select_p<64, 1>(a, nmax, units, gb, stream, dependent);
}

}  // namespace cva
