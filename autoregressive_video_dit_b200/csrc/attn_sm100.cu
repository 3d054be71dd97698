// Step 5 of the per-chunk path: block-sparse flash attention on sm_100a.
//
// "Light Forcing", section 2.2 (execution): attention runs only over the
// picked frame-block pairs, here together with every token of the current
// chunk; its cost is independent of how long the history is.
//
// A CTA owns one SM and works on two 128-row query tiles of one (batch,
// head) at once, in two independent lanes (A and B). Each lane has its own
// key list, its own Q, K and V tiles in shared memory and its own S and O
// accumulators in tensor memory (4 x 128 columns). A key list is a list of
// 64-row key units: the union of the picked history blocks of the lane's
// query blocks (two 64-token query blocks share a tile when blk = 64; a unit
// carries a 2-bit mask of the query blocks that picked it), followed by the
// current chunk's blocks. Pairs of units form 128-key tiles.
//
// Roles (384 threads):
//   warps 0-3 / 4-7: softmax of lane A / B; thread i owns query row i
//     (TMEM lane i). One tensor-memory load brings the 128 scores of a tile
//     into registers; masks, row maximum (3-input max), exp2 on the MUFU in
//     fp32 with packed f32x2 arithmetic, bf16 P written back over the S
//     columns. O is rescaled in tensor memory only when the row maximum grows
//     by more than 2^8. Finally O is normalised into bf16.
//   warp 8 (one lane): TMA producer. Q once per lane; then per key tile K
//     into the lane's K slot (free once S of the previous tile completed) and
//     V into its V slot (free once PV completed), gathered by block index
//     with one 64-row box per unit and 64-column chunk, 128-byte swizzle.
//     No multicast.
//   warp 9 (one lane): tcgen05.mma issuer, interleaving the lanes:
//     PV_A(n), S_A(n+1), PV_B(n), S_B(n+1), ... so that one lane's MMAs run
//     while the other lane's softmax does.
// Every wait is bounded: on timeout the CTA latches CVA_DEV_TIMEOUT, all
// roles leave their loops, in-flight copies and MMAs are drained with a
// bounded wait and the tensor memory is released.
#include <cudaTypedefs.h>
#include <math.h>

#include "kernels.cuh"

namespace cva {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kLanes = 2;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
// 12 warps: registers are granted per group of four warps, so warps 10 and
// 11 cost nothing extra; they only join the final barrier.
constexpr int kAttnThreads = 384;
constexpr uint32_t kTmemCols = 512;   // lane x: S at 256x (P aliased onto it), O at 256x + 128
constexpr uint32_t kOCol = 128;

template <int D>
struct AttnSmem {
  static constexpr int kChunkBytes = 128 * 128;  // 128 rows x 128 B: one 64-column chunk
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kChunks * kChunkBytes;  // a Q, K or V tile
  static constexpr int kQ = 0;                              // lane x at + x * tile
  static constexpr int kK = kQ + kLanes * kTileBytes;
  static constexpr int kV = kK + kLanes * kTileBytes;
  static constexpr int kEnt = kV + kLanes * kTileBytes;     // lane x at + x * entries
  static constexpr int kBm = kEnt + kLanes * kAttnMaxEntries * 4;
  static constexpr int kScan = kBm + 2 * kAttnMaxBitmapWords * 4;
  static constexpr int kBar = kScan + kAttnMaxBitmapWords * 4;
  static constexpr int kMisc = kBar + 32 * 8;
  static constexpr int kBytes = kMisc + 64;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024 B
};

// Barrier slots of lane x: 8 * x + slot.
enum : int { kBarQ = 0, kBarKFull = 1, kBarVFull = 2, kBarKEmpty = 3, kBarVEmpty = 4, kBarSFull = 5,
             kBarPFull = 6, kBarODone = 7 };
constexpr int kBarDrain = 16;

// Above this growth of the row maximum (log2 units) O is rescaled; below
// it the stale maximum is kept, so P <= 2^8.
constexpr float kRescaleThreshold = 8.0f;

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// A wait with its own limit that ignores the abort flag (used while draining).
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) return;  // 200 ms
  }
}

// Key unit: (row64 << 16) | (valid << 8) | mask. row64 indexes 64-row
// groups inside one (batch, head) slice of the cache.
__device__ __forceinline__ uint32_t make_unit(int row64, int valid, uint32_t mask) {
  return ((uint32_t)row64 << 16) | ((uint32_t)valid << 8) | mask;
}

__device__ __forceinline__ int unit_valid(int block_valid, int u) {
  int v = block_valid - 64 * u;
  return v < 0 ? 0 : (v > 64 ? 64 : v);
}

// Builds the tile's key-unit list in smem; returns the number of units.
// Must be called by all threads of the CTA.
__device__ int build_units(const AttnArgs& a, int m, int bh, uint32_t* ents, uint32_t* bm,
                           uint32_t* wcnt, int* total_slot) {
  const Dims& d = a.d;
  const int tid = threadIdx.x;
  const int upb = d.blk / 64;
  const int rows64_slot = d.T_pad / 64;
  int hist = 0;
  if (a.F > 0) {
    if (a.block_idx == nullptr) {
      hist = a.F * d.nb * upb;
      for (int i = tid; i < hist; i += kAttnThreads) {
        const int br = i / upb, u = i - br * upb;
        const int fp = br / d.nb, j = br - fp * d.nb;
        const int slot = (a.t_lo + fp) % a.W;
        const int vb = (j == d.nb - 1) ? d.tail : d.blk;
        ents[i] = make_unit(slot * rows64_slot + j * upb + u, unit_valid(vb, u), 3u);
      }
    } else {
      const int nbits = a.F * d.nb;
      const int nw = (nbits + 31) >> 5;
      for (int i = tid; i < nw; i += kAttnThreads) {
        bm[i] = 0u;
        bm[kAttnMaxBitmapWords + i] = 0u;
      }
      __syncthreads();
      const int nq = (d.blk == 64) ? 2 : 1;
      for (int q = 0; q < nq; ++q) {
        const int qb = (d.blk == 64) ? 2 * m + q : m;
        if (qb >= d.NQB) continue;
        const size_t u = (size_t)bh * d.NQB + qb;
        int cnt = a.block_cnt ? a.block_cnt[u] : a.k_b_max;
        if (cnt < 0 || cnt > a.k_b_max) {
          if (tid == 0) latch_error(a.err, CVA_DEV_BAD_COUNT);
          cnt = cnt < 0 ? 0 : a.k_b_max;
        }
        const int32_t* lst = a.block_idx + u * a.k_b_max;
        for (int i = tid; i < cnt; i += kAttnThreads) {
          const int id = lst[i];
          const int rel = id - a.t_lo * d.nb;
          if (id < 0 || rel < 0 || rel >= nbits) {
            latch_error(a.err, CVA_DEV_BAD_INDEX);
            continue;
          }
          atomicOr(&bm[q * kAttnMaxBitmapWords + (rel >> 5)], 1u << (rel & 31));
        }
      }
      __syncthreads();
      for (int w = tid; w < nw; w += kAttnThreads)
        wcnt[w] = __popc(bm[w] | bm[kAttnMaxBitmapWords + w]) * upb;
      __syncthreads();
      if (tid < 32) {  // exclusive scan of the per-word counts
        int carry = 0;
        for (int base = 0; base < nw; base += 32) {
          const int w = base + tid;
          const int v = (w < nw) ? (int)wcnt[w] : 0;
          int incl = v;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (tid >= o) incl += t;
          }
          if (w < nw) wcnt[w] = (uint32_t)(carry + incl - v);
          carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (tid == 0) *total_slot = carry;
      }
      __syncthreads();
      hist = *total_slot;
      for (int w = tid; w < nw; w += kAttnThreads) {
        const uint32_t b0 = bm[w], b1 = bm[kAttnMaxBitmapWords + w];
        uint32_t any = b0 | b1;
        int pos = (int)wcnt[w];
        while (any) {
          const int bit = __ffs(any) - 1;
          any &= any - 1u;
          const int rel = w * 32 + bit;
          const int fp = rel / d.nb, j = rel - fp * d.nb;
          const int slot = (a.t_lo + fp) % a.W;
          const uint32_t mask =
              (d.blk == 64) ? (((b0 >> bit) & 1u) | (((b1 >> bit) & 1u) << 1)) : 3u;
          const int vb = (j == d.nb - 1) ? d.tail : d.blk;
          for (int u = 0; u < upb; ++u)
            ents[pos++] = make_unit(slot * rows64_slot + j * upb + u, unit_valid(vb, u), mask);
        }
      }
    }
  }
  const int cur = d.Fc * d.nb * upb;
  for (int i = tid; i < cur; i += kAttnThreads) {
    const int br = i / upb, u = i - br * upb;
    const int f = br / d.nb, j = br - f * d.nb;
    const int slot = (a.t0 + f) % a.W;
    const int vb = (j == d.nb - 1) ? d.tail : d.blk;
    ents[hist + i] = make_unit(slot * rows64_slot + j * upb + u, unit_valid(vb, u), 3u);
  }
  __syncthreads();
  return hist + cur;
}

template <int D>
__device__ __forceinline__ void issue_s(uint32_t s_tmem, uint32_t q_addr, uint32_t k_addr) {
  constexpr uint32_t kIdS = idesc_bf16_f32(kBM, kBN, 0, 0);  // Q, K both K-major
#pragma unroll
  for (int k = 0; k < D / 16; ++k) {
    const uint32_t off = (uint32_t)((k >> 2) * AttnSmem<D>::kChunkBytes + (k & 3) * 32);
    mma_ss(s_tmem, smem_desc_sw128(q_addr + off, 16, 1024), smem_desc_sw128(k_addr + off, 16, 1024),
           kIdS, k > 0 ? 1u : 0u);
  }
}

template <int D>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_addr,
                                         bool accumulate) {
  constexpr uint32_t kIdO = idesc_bf16_f32(kBM, D, 0, 1);    // P (tmem), V MN-major
#pragma unroll
  for (int k = 0; k < kBN / 16; ++k) {
    mma_ts(o_tmem, p_tmem + (uint32_t)(k * 8),
           smem_desc_sw128(v_addr + (uint32_t)(k * 2048), AttnSmem<D>::kChunkBytes, 1024), kIdO,
           (accumulate || k > 0) ? 1u : 0u);
  }
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  using L = AttnSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int bh = blockIdx.y;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  int* total_slot = reinterpret_cast<int*>(smem + L::kMisc + 8);
  int m_of[kLanes];
  for (int x = 0; x < kLanes; ++x) m_of[x] = kLanes * blockIdx.x + x;

  if (tid == 0) {
    for (int x = 0; x < kLanes; ++x) {
      uint64_t* b = bar + 8 * x;
      mbar_init(&b[kBarQ], 1);
      mbar_init(&b[kBarKFull], 1);
      mbar_init(&b[kBarVFull], 1);
      mbar_init(&b[kBarKEmpty], 1);
      mbar_init(&b[kBarVEmpty], 1);
      mbar_init(&b[kBarSFull], 1);
      mbar_init(&b[kBarPFull], 128);
      mbar_init(&b[kBarODone], 1);
    }
    mbar_init(&bar[kBarDrain], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  int N[kLanes];
  for (int x = 0; x < kLanes; ++x) {
    int E = 0;
    if (m_of[x] < a.MT)
      E = build_units(a, m_of[x], bh, reinterpret_cast<uint32_t*>(smem + L::kEnt) + x * kAttnMaxEntries,
                      reinterpret_cast<uint32_t*>(smem + L::kBm), reinterpret_cast<uint32_t*>(smem + L::kScan),
                      total_slot);
    N[x] = E;  // units for now; tiles below
  }
  int E_of[kLanes];
  for (int x = 0; x < kLanes; ++x) {
    E_of[x] = N[x];
    N[x] = (N[x] + 1) >> 1;  // 128-key tiles
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int k_issued[kLanes] = {0, 0}, v_issued[kLanes] = {0, 0};
      auto load_kv = [&](int x, int n, bool is_v) {
        const uint32_t* ents = reinterpret_cast<const uint32_t*>(smem + L::kEnt) + x * kAttnMaxEntries;
        const uint32_t e0 = ents[2 * n];
        const uint32_t e1 = (2 * n + 1 < E_of[x]) ? ents[2 * n + 1] : (e0 & 0xFFFF0000u);
        const int r0 = (int)(e0 >> 16) * 64;
        const int r1 = (int)(e1 >> 16) * 64;
        uint64_t* full = &bar[8 * x + (is_v ? kBarVFull : kBarKFull)];
        uint8_t* dst = smem + (is_v ? L::kV : L::kK) + x * L::kTileBytes;
        const CUtensorMap* map = is_v ? &tmV : &tmK;
        mbar_arrive_expect_tx(full, L::kTileBytes);
        for (int c = 0; c < L::kChunks; ++c) {
          tma_load_3d(dst + c * L::kChunkBytes, map, full, c * 64, r0, bh);
          tma_load_3d(dst + c * L::kChunkBytes + 8192, map, full, c * 64, r1, bh);
        }
      };
      bool ok = true;
      for (int x = 0; x < kLanes; ++x) {
        if (N[x] == 0) continue;
        mbar_arrive_expect_tx(&bar[8 * x + kBarQ], L::kTileBytes);
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_3d(smem + L::kQ + x * L::kTileBytes + c * L::kChunkBytes, &tmQ, &bar[8 * x + kBarQ],
                      c * 64, m_of[x] * kBM, bh);
        load_kv(x, 0, false);
        k_issued[x] = 1;
        load_kv(x, 0, true);
        v_issued[x] = 1;
      }
      const int n_max = N[0] > N[1] ? N[0] : N[1];
      for (int n = 1; ok && n < n_max; ++n) {
        // K of tile n once S(n-1) completed, then V once PV(n-1) completed,
        // lane A before lane B: the order in which those events happen.
        for (int x = 0; ok && x < kLanes; ++x) {
          if (n >= N[x]) continue;
          if (!mbar_wait(&bar[8 * x + kBarKEmpty], (n - 1) & 1, abort_flag, a.err)) { ok = false; break; }
          load_kv(x, n, false);
          k_issued[x] = n + 1;
        }
        for (int x = 0; ok && x < kLanes; ++x) {
          if (n >= N[x]) continue;
          if (!mbar_wait(&bar[8 * x + kBarVEmpty], (n - 1) & 1, abort_flag, a.err)) { ok = false; break; }
          load_kv(x, n, true);
          v_issued[x] = n + 1;
        }
      }
      if (*abort_flag) {  // let copies in flight land before the CTA exits
        for (int x = 0; x < kLanes; ++x) {
          if (N[x] == 0) continue;
          mbar_wait_drain(&bar[8 * x + kBarQ], 0);
          if (k_issued[x]) mbar_wait_drain(&bar[8 * x + kBarKFull], (k_issued[x] - 1) & 1);
          if (v_issued[x]) mbar_wait_drain(&bar[8 * x + kBarVFull], (v_issued[x] - 1) & 1);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(smem + L::kQ);
      const uint32_t k_addr = smem_u32(smem + L::kK);
      const uint32_t v_addr = smem_u32(smem + L::kV);
      bool ok = true;
      for (int x = 0; ok && x < kLanes; ++x) {
        if (N[x] == 0) continue;
        uint64_t* b = bar + 8 * x;
        ok = mbar_wait(&b[kBarQ], 0, abort_flag, a.err) && mbar_wait(&b[kBarKFull], 0, abort_flag, a.err);
        if (!ok) break;
        tc_fence_after();
        issue_s<D>(tmem + 256u * x, q_addr + x * L::kTileBytes, k_addr + x * L::kTileBytes);
        mma_commit(&b[kBarSFull]);
        mma_commit(&b[kBarKEmpty]);
      }
      int np[kLanes] = {0, 0};
      while (ok && (np[0] < N[0] || np[1] < N[1])) {
        for (int x = 0; ok && x < kLanes; ++x) {
          const int n = np[x];
          if (n >= N[x]) continue;
          uint64_t* b = bar + 8 * x;
          if (!mbar_wait(&b[kBarPFull], n & 1, abort_flag, a.err) ||
              !mbar_wait(&b[kBarVFull], n & 1, abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
          issue_pv<D>(tmem + 256u * x + kOCol, tmem + 256u * x, v_addr + x * L::kTileBytes, n > 0);
          mma_commit(&b[kBarVEmpty]);
          if (n + 1 == N[x]) mma_commit(&b[kBarODone]);  // O final: the epilogue's single wait
          np[x] = n + 1;
          if (n + 1 < N[x]) {
            // S(n+1) overwrites the columns holding P(n); PV(n) was issued
            // before it by this thread and tcgen05.mma executes in issue
            // order. Its commit also covers PV(n): once S(n+1) is reported
            // complete, O holds PV(0..n) and may be rescaled.
            if (!mbar_wait(&b[kBarKFull], (n + 1) & 1, abort_flag, a.err)) { ok = false; break; }
            tc_fence_after();
            issue_s<D>(tmem + 256u * x, q_addr + x * L::kTileBytes, k_addr + x * L::kTileBytes);
            mma_commit(&b[kBarSFull]);
            mma_commit(&b[kBarKEmpty]);
          }
        }
      }
      mma_commit(&bar[kBarDrain]);
      mbar_wait_drain(&bar[kBarDrain], 0);
    }
  } else if (warp < kLanes * 4) {
    // ------------------------------------------------------------ softmax
    const Dims& d = a.d;
    const int x = warp >> 2;           // lane (query tile) of this warp group
    const int r = tid & 127;           // query row of the tile = TMEM lane
    const int Nx = N[x];
    const int Ex = E_of[x];
    const uint32_t* ents = reinterpret_cast<const uint32_t*>(smem + L::kEnt) + x * kAttnMaxEntries;
    uint64_t* b = bar + 8 * x;
    const uint32_t trow = tmem + 256u * x + ((uint32_t)((warp & 3) * 32) << 16);
    const int qsel = r >> 6;   // warp-uniform
    const float sc = a.scale_log2;
    float m_used = -INFINITY;  // running maximum in scaled log2 units (possibly stale by < 8)
    float l_run = 0.f;
    bool ok = Nx > 0;
    for (int n = 0; ok && n < Nx; ++n) {
      ok = mbar_wait(&b[kBarSFull], n & 1, abort_flag, a.err);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t s[4][32];
#pragma unroll
      for (int i = 0; i < 4; ++i) tmem_ld32(trow + (uint32_t)(32 * i), s[i]);
      const uint32_t e0 = ents[2 * n];
      const uint32_t e1 = (2 * n + 1 < Ex) ? ents[2 * n + 1] : 0u;
      const int lim0 = ((e0 >> qsel) & 1u) ? (int)((e0 >> 8) & 0xFFu) : 0;
      const int lim1 = ((e1 >> qsel) & 1u) ? (int)((e1 >> 8) & 0xFFu) : 0;
      const bool full = (lim0 == 64) && (lim1 == 64);   // warp-uniform
      tmem_wait_ld();
      if (!full) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int lim = i < 2 ? lim0 - 32 * i : lim1 - 32 * (i - 2);
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c >= lim) s[i][c] = __float_as_uint(-INFINITY);
        }
      }
      float ma = -INFINITY, mb = -INFINITY;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          ma = max3f(ma, __uint_as_float(s[i][c]), __uint_as_float(s[i][c + 1]));
          mb = max3f(mb, __uint_as_float(s[i][c + 2]), __uint_as_float(s[i][c + 3]));
        }
      }
      const float mt = fmaxf(ma, mb) * sc;  // -inf when nothing is valid
      const bool need = mt > m_used + kRescaleThreshold || (m_used == -INFINITY && mt > -INFINITY);
      if (__any_sync(0xFFFFFFFFu, need)) {
        const float m_new = need ? mt : m_used;
        const float alpha = (m_used == -INFINITY) ? 0.f : fast_exp2(m_used - m_new);
        if (n > 0) {
          // O holds PV(0..n-1): the commit of S(n) covered PV(n-1).
#pragma unroll 1
          for (int i = 0; i < D / 16; ++i) {
            uint32_t o[16];
            tmem_ld16(trow + kOCol + (uint32_t)(16 * i), o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st16(trow + kOCol + (uint32_t)(16 * i), o);
          }
        }
        l_run *= alpha;
        m_used = m_new;
      }
      const float base = (m_used == -INFINITY) ? 0.f : m_used;
      const float2 sc2 = make_float2(sc, sc);
      const float2 nb2 = make_float2(-base, -base);
      float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float2 xv = ffma2(make_float2(__uint_as_float(s[h][2 * q]), __uint_as_float(s[h][2 * q + 1])),
                                  sc2, nb2);
          const float2 p = make_float2(fast_exp2(xv.x), fast_exp2(xv.y));
          if (q & 1) acc1 = fadd2(acc1, p);
          else acc0 = fadd2(acc0, p);
          pk[q] = cvt_bf16x2(p.x, p.y);
        }
        tmem_st16(trow + (uint32_t)(16 * h), pk);
      }
      l_run += (acc0.x + acc0.y) + (acc1.x + acc1.y);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&b[kBarPFull]);
    }
    // ------------------------------------------------------------ epilogue
    if (ok) {
      ok = mbar_wait(&b[kBarODone], 0, abort_flag, a.err);
      ok = __all_sync(0xFFFFFFFFu, ok);
    }
    if (ok) {
      tc_fence_after();
      const int pr = m_of[x] * kBM + r;  // row in the padded chunk
      const int f = pr / d.T_pad;
      const int rr = pr - f * d.T_pad;
      const bool row_ok = (f < d.Fc) && (rr < d.T_f);
      const int bb = bh / d.H;
      const int h = bh - bb * d.H;
      const size_t n_tok = (size_t)f * d.T_f + rr;
      const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
      uint16_t* orow = a.out + (((size_t)bb * d.Lq + n_tok) * d.H + h) * D;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        uint32_t o[32];
        tmem_ld32(trow + kOCol + (uint32_t)(32 * i), o);
        tmem_wait_ld();
        if (row_ok) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            pk[c] = cvt_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * i);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      if (row_ok && a.lse)
        a.lse[(size_t)bh * d.Lq + n_tok] = (m_used + log2f(l_run)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- host side --------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3D bf16 map over [d2][d1][d0] (d0 innermost), box (64 columns, box1 rows), 128 B swizzle.
static bool make_map(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                     uint32_t box1) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {64, box1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                         strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D>
static cudaError_t launch_attention_d(const AttnArgs& a, const CUtensorMap& mq, const CUtensorMap& mk,
                                      const CUtensorMap& mv, cudaStream_t stream) {
  using L = AttnSmem<D>;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       L::kAlloc);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  dim3 grid((a.MT + kLanes - 1) / kLanes, a.d.B * a.d.H);
  attn_fwd_kernel<D><<<grid, kAttnThreads, L::kAlloc, stream>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

cudaError_t launch_attention(const AttnArgs& a, const void* q_rot, const void* cache_k,
                             const void* cache_v, cudaStream_t stream, const char** why) {
  const Dims& d = a.d;
  CUtensorMap mq, mk, mv;
  const uint64_t bh = (uint64_t)d.B * d.H;
  if (!make_map(&mq, q_rot, d.D, (uint64_t)d.Fc * d.T_pad, bh, 128) ||
      !make_map(&mk, cache_k, d.D, (uint64_t)a.W * d.T_pad, bh, 64) ||
      !make_map(&mv, cache_v, d.D, (uint64_t)a.W * d.T_pad, bh, 64)) {
    *why = "cuTensorMapEncodeTiled failed (driver entry point or tensor shape)";
    return cudaErrorInvalidValue;
  }
  return d.D == 128 ? launch_attention_d<128>(a, mq, mk, mv, stream)
                    : launch_attention_d<64>(a, mq, mk, mv, stream);
}

}  // namespace cva
