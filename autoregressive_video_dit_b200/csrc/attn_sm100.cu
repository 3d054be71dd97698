// Step 5 of the per-chunk path: block-sparse flash attention on sm_100a.
//
// "Light Forcing", section 2.2 (execution): attention runs only over the
// picked frame-block pairs, here together with every token of the current
// chunk; its cost is independent of how long the history is.
//
// A CTA owns one SM and one 128-row query tile of one (batch, head). Its
// keys come as a stream of 64-row key units, two per 128-key tile: the
// current chunk's blocks, then the union of the history blocks its query
// blocks picked (two 64-token query blocks share a tile when blk = 64; a
// unit's mask says which of them picked it); an odd count is padded with an
// empty unit.
//
// Tensor memory holds one output accumulator O (columns 0 .. D-1) and three
// score buffers S0, S1, S2 (128 fp32 columns each at 128, 256, 384; P is
// written back over the first 64 columns of its own scores). Key tile i goes
// to buffer i mod 3, so the scores of the next two tiles are computed while
// the softmax works on tile i: the chain S(i) -> softmax(i) -> PV(i) ->
// S(i+3) has three links in flight and the tensor core does not wait for
// one softmax to finish before the next tile's scores.
//
// The softmax of all tiles shares one running maximum per query row, so that
// every PV accumulates into the one O: the online softmax keeps a reference
// maximum m that only moves up, and only when a tile's row maximum exceeds it
// by more than 2^8 (in the exponent); P = 2^(s/sqrt(D) log2 e - m) <= 2^8
// otherwise. Tile i's warp needs m after tile i-1 before it can fix P(i): the
// two warps of a row range hand m over through shared memory and an mbarrier
// per direction, once per tile, right after their row maxima (early in the
// tile). When m moves up at tile i the warp rescales its rows of O, after
// PV(i-1) completed and before it releases P(i) (so before PV(i) is issued).
//
// Roles (384 threads):
//   warps 0-3 / 4-7: softmax of the even / odd key tiles. Warps w and w + 4
//     own query rows 32 (w mod 4) .. + 31 (TMEM lanes; thread = row). Masks,
//     row maximum (3-input max), the hand-over of m, exp2 on the MUFU in fp32
//     with packed f32x2 arithmetic, bf16 P written back over the S columns.
//     Each warp keeps its own row sum relative to the m it last saw; at the
//     end the pair merges the two sums and writes bf16 O (each warp half of
//     the columns).
//   warp 8 (one lane): TMA producer. Q once, then K and V of every tile in
//     the order the MMAs consume them, K into ring slot t mod 2 and V into
//     slot t mod 3, each as soon as its slot is free, gathered by block index
//     with one 64-row box per unit and 64-column chunk, 128-byte swizzle. No
//     multicast.
//   warp 9 (one lane): tcgen05.mma issuer, in the fixed order S(0), S(1),
//     S(2), PV(0), S(3), PV(1), S(4), ...
//   warps 10-11: frame means of the chunk's new cache frames (fused call).
// Every wait is bounded: on timeout the CTA latches CVA_DEV_TIMEOUT, all
// roles leave their loops, in-flight copies and MMAs are drained with a
// bounded wait and the tensor memory is released.
//
// Tail split: the tiles of the last, partial wave of CTAs would leave most
// SMs idle for a whole tile's time. Given scratch, the host cuts each of
// them into `pieces` contiguous ranges of its key tiles; a piece writes its
// unnormalised O, running maximum and sum, and attn_merge_kernel combines
// the pieces of a tile (flash-decoding style) into bf16 O and LSE.
#include <cudaTypedefs.h>
#include <math.h>

#include <type_traits>

#include "kernels.cuh"

namespace cva {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kKStages = 2;   // K ring slots (tile t in slot t mod 2)
constexpr int kVStages = 3;   // V ring slots (tile t in slot t mod 3)
constexpr int kSBufs = 3;     // score buffers in tensor memory
constexpr int kSoftmaxWarps = 8;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
// 12 warps in three warpgroups: the two softmax warpgroups, then the
// producer, the MMA issuer and two warps for the frame means. The launch
// grants 168 registers a thread (three warps per scheduler); after the key
// stream is built the third warpgroup gives registers back (setmaxnreg.dec
// to kRegsOther) and the softmax warpgroups take them (setmaxnreg.inc to
// kRegsSoftmax): 2 * 128 * 224 + 128 * 56 = 384 * 168, exactly the launch's
// registers, so the increase always completes.
constexpr int kAttnThreads = 384;
constexpr int kRegsSoftmax = 224;
constexpr int kRegsOther = 56;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther <= kAttnThreads * 168, "register split");
constexpr uint32_t kTmemCols = 512;   // O at 0, S0 at 128, S1 at 256, S2 at 384
constexpr uint32_t kOCol = 0;
constexpr uint32_t kSCol = 128;

template <int D>
struct AttnSmem {
  static constexpr int kChunkBytes = 128 * 128;  // 128 rows x 128 B: one 64-column chunk
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kChunks * kChunkBytes;  // a Q, K or V tile
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;                // slot s at + s * tile
  static constexpr int kV = kK + kKStages * kTileBytes;
  static constexpr int kEnt = kV + kVStages * kTileBytes;
  // softmax epilogue exchange: (max, sum) [2 parities][128 rows], flags [2][4];
  // then the hand-over of the running maximum: [128 rows] floats
  static constexpr int kRed = kEnt + kAttnMaxEntries * 4;
  static constexpr int kHand = kRed + 2 * 128 * 8 + 2 * 4 * 4;
  static constexpr int kBar = kHand + 128 * 4;
  static constexpr int kMisc = kBar + 32 * 8;
  static constexpr int kBytes = kMisc + 64;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024 B
  // While the key list is built, its bitmaps and counts live in the V ring.
  static constexpr int kBm = kV;                                   // 2 bitmaps
  static constexpr int kCnt = kBm + 2 * kAttnMaxBitmapWords * 4;   // word offsets, total
  static_assert((3 * kAttnMaxBitmapWords + 1) * 4 <= kVStages * kTileBytes, "build scratch");
  static_assert(kAlloc <= 227 * 1024, "shared memory");
};

// Barriers: S buffer b full (3; S(j) completing also frees K slot j mod 2);
// K ring slots full (2); V ring slots full -- V(t) landed and P(t) written --
// and free (3 each; V slot t mod 3
// frees when PV(t) completes, so it also tells that PV(t) is done); Q; O
// final; one for draining the tensor pipe; the hand-over of the running
// maximum per row range: [quarter][0] even -> odd tiles, [quarter][1] odd ->
// even tiles.
constexpr int kBarSFull = 0, kBarKFull = 3, kBarVFull = 5, kBarVEmpty = 8, kBarQ = 11,
              kBarODone = 12, kBarDrain = 13, kBarHand = 14;  // .. 21

// Above this growth of the row maximum (log2 units) O is rescaled; below
// it the stale maximum is kept, so P <= 2^8.
constexpr float kRescaleThreshold = 8.0f;


__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Barrier of the two warps that share a row range (ids 1..4; 0 is __syncthreads).
__device__ __forceinline__ void pair_sync(int quarter) {
  asm volatile("bar.sync %0, 64;" ::"r"(quarter + 1) : "memory");
}

// A wait with its own limit that ignores the abort flag (used while draining).
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) return;  // 200 ms
  }
}

// Key unit: (row64 << 16) | (valid << 8) | mask. row64 indexes 64-row
// groups inside one (batch, head) slice of the cache; an empty unit (row 0,
// valid 0, mask 0) pads a section to whole tiles.
__device__ __forceinline__ uint32_t make_unit(int row64, int valid, uint32_t mask) {
  return ((uint32_t)row64 << 16) | ((uint32_t)valid << 8) | mask;
}

__device__ __forceinline__ int unit_valid(int block_valid, int u) {
  int v = block_valid - 64 * u;
  return v < 0 ? 0 : (v > 64 ? 64 : v);
}

// Query block in rows [64 half, 64 half + 64) of tile m of head bh (64-row blocks).
__device__ __forceinline__ int tile_qb(const AttnArgs& a, int bh, int m, int half) {
  return a.qpair ? a.qpair[((size_t)bh * a.MT + m) * 2 + half] : 2 * m + half;
}
// Row of the padded chunk held in row r of tile m (-1: none).
__device__ __forceinline__ int tile_row(const AttnArgs& a, int bh, int m, int r) {
  if (!a.qpair) return m * kBM + r;
  const int qb = a.qpair[((size_t)bh * a.MT + m) * 2 + (r >> 6)];
  return qb < 0 ? -1 : qb * 64 + (r & 63);
}

// Builds the key stream of query tile m0 of head bh into `ents`, two 64-row
// units per key tile, and returns its number of key tiles; must be called
// by all threads of the CTA. Dense: the history units, then the current
// chunk's, padded to a whole tile. Sparse: the current chunk's units padded
// to a whole tile, then the union of the selected blocks of the tile's two
// query blocks in ascending order, each unit with a mask of which query
// block selected it (bit q: rows [64 q, 64 q + 64)). Every thread handles
// its own list entries and bitmap bits; no step is serial over the list.
__device__ int build_stream(const AttnArgs& a, int m0, int bh, uint32_t* ents, uint32_t* bm,
                            uint32_t* cnt) {
  constexpr int kW = kAttnMaxBitmapWords;
  const Dims& d = a.d;
  const int tid = threadIdx.x;
  const int upb = d.blk / 64;
  const int rows64_slot = d.T_pad / 64;
  const int nbits = a.F * d.nb;
  const bool sparse = a.F > 0 && a.block_idx != nullptr;
  const int cur = d.Fc * d.nb * upb;
  const int hist = (a.F > 0 && !sparse) ? nbits * upb : 0;   // dense history units
  const int c0 = sparse ? 0 : hist;                          // first unit of the current chunk
  for (int i = tid; i < hist; i += kAttnThreads) {
    const int br = i / upb, u = i - br * upb;
    const int fp = br / d.nb, j = br - fp * d.nb;
    const int slot = (a.t_lo + fp) % a.W;
    const int vb = (j == d.nb - 1) ? d.tail : d.blk;
    ents[i] = make_unit(slot * rows64_slot + j * upb + u, unit_valid(vb, u), 0x3u);
  }
  for (int i = tid; i < cur; i += kAttnThreads) {
    const int br = i / upb, u = i - br * upb;
    const int f = br / d.nb, j = br - f * d.nb;
    const int slot = (a.t0 + f) % a.W;
    const int vb = (j == d.nb - 1) ? d.tail : d.blk;
    ents[c0 + i] = make_unit(slot * rows64_slot + j * upb + u, unit_valid(vb, u), 0x3u);
  }
  if (tid == 0 && ((c0 + cur) & 1)) ents[c0 + cur] = 0u;
  const int lead = (c0 + cur + 1) >> 1;   // key tiles before the sparse section
  if (!sparse) {
    __syncthreads();
    return lead;
  }
  const int nw = (nbits + 31) >> 5;
  const int nq = (d.blk == 64) ? 2 : 1;
  const int kbm = a.k_b_max;
  for (int i = tid; i < 2 * kW; i += kAttnThreads) bm[i] = 0u;
  __syncthreads();
  for (int i = tid; i < nq * kbm; i += kAttnThreads) {
    const int q = i >= kbm ? 1 : 0;
    const int k = i - q * kbm;
    const int qb = (d.blk == 64) ? tile_qb(a, bh, m0, q) : m0;
    if (qb < 0 || qb >= d.NQB) continue;
    const size_t u = (size_t)bh * d.NQB + qb;
    const int id = a.block_idx[u * kbm + k];   // in the list's storage whatever the count
    int c = a.block_cnt ? a.block_cnt[u] : kbm;
    if (c < 0 || c > kbm) {
      if (k == 0) latch_error(a.err, CVA_DEV_BAD_COUNT);
      c = c < 0 ? 0 : kbm;
    }
    if (k >= c) continue;
    const int rel = id - a.t_lo * d.nb;
    if (id < 0 || rel < 0 || rel >= nbits) {
      latch_error(a.err, CVA_DEV_BAD_INDEX);
      continue;
    }
    atomicOr(&bm[q * kW + (rel >> 5)], 1u << (rel & 31));
  }
  __syncthreads();
  if (tid < 32) {  // exclusive scan of the units per bitmap word
    int carry = 0;
    for (int base = 0; base < nw; base += 32) {
      const int w = base + tid;
      const int v = (w < nw) ? __popc(bm[w] | bm[kW + w]) * upb : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (tid >= o) incl += t;
      }
      if (w < nw) cnt[w] = (uint32_t)(carry + incl - v);
      carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (tid == 0) cnt[kW] = (uint32_t)carry;
  }
  __syncthreads();
  const int n_sp = (int)cnt[kW];
  uint32_t* sp = ents + 2 * lead;
  for (int rel = tid; rel < nbits; rel += kAttnThreads) {
    const int w = rel >> 5, bit = rel & 31;
    const uint32_t b0 = bm[w], b1 = bm[kW + w], any = b0 | b1;
    if (!((any >> bit) & 1u)) continue;
    const int pos = (int)cnt[w] + __popc(any & ((1u << bit) - 1u)) * upb;
    const uint32_t mask = nq == 1 ? 0x3u : (((b0 >> bit) & 1u) | (((b1 >> bit) & 1u) << 1));
    const int fp = rel / d.nb, j = rel - fp * d.nb;
    const int slot = (a.t_lo + fp) % a.W;
    const int vb = (j == d.nb - 1) ? d.tail : d.blk;
    for (int u = 0; u < upb; ++u)
      sp[pos + u] = make_unit(slot * rows64_slot + j * upb + u, unit_valid(vb, u), mask);
  }
  if (tid == 0 && (n_sp & 1)) sp[n_sp] = 0u;
  __syncthreads();
  return lead + ((n_sp + 1) >> 1);
}

// The MMAs of one key tile, from shared-memory descriptors computed once per
// CTA: the descriptor's start address field is the byte address / 16 in its
// low 14 bits, and every operand lies below 256 KB, so the k-th step's
// descriptor is the base plus a compile-time constant. (One thread issues
// all MMAs; keeping its instruction stream short and free of dependent
// chains is what lets it keep up with the tensor core.)
template <int D>
__device__ __forceinline__ void issue_s(uint32_t s_tmem, uint64_t q_desc, uint64_t k_desc) {
  constexpr uint32_t kIdS = idesc_bf16_f32(kBM, kBN, 0, 0);  // Q, K both K-major
#pragma unroll
  for (int k = 0; k < D / 16; ++k) {
    const uint64_t off = (uint64_t)(((k >> 2) * AttnSmem<D>::kChunkBytes + (k & 3) * 32) >> 4);
    mma_ss(s_tmem, q_desc + off, k_desc + off, kIdS, k > 0 ? 1u : 0u);
  }
}

template <int D>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint64_t v_desc,
                                         bool accumulate) {
  constexpr uint32_t kIdO = idesc_bf16_f32(kBM, D, 0, 1);    // P (tmem), V MN-major
#pragma unroll
  for (int k = 0; k < kBN / 16; ++k)
    mma_ts(o_tmem, p_tmem + (uint32_t)(k * 8), v_desc + (uint64_t)((k * 2048) >> 4), kIdO,
           (accumulate || k > 0) ? 1u : 0u);
}


template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  using L = AttnSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  griddep_launch_dependents();
  // Work item: a whole tile, or one key-range piece of a tail tile.
  int tile = blockIdx.x, piece = 0, slot = -1;
  if (tile >= a.Qf) {
    const int k = tile - a.Qf;
    tile = a.Qf + k / a.pieces;
    piece = k % a.pieces;
    slot = k;                  // partial-result slot
  }
  const int bh = tile / a.MT;
  const int m = tile - bh * a.MT;  // query tile
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  uint32_t* ents = reinterpret_cast<uint32_t*>(smem + L::kEnt);

  if (tid == 0) {
    for (int s = 0; s < kSBufs; ++s) mbar_init(&bar[kBarSFull + s], 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bar[kBarKFull + s], 1);
    }
    // VFull[s] completes when V(i) landed in slot s AND P(i) was written
    // (i mod 3 == s for both): the producer's arrive with the byte count plus
    // the 128 softmax threads of tile i, so the MMA warp waits once per PV.
    static_assert(kVStages == kSBufs, "V slot and score buffer share an index");
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bar[kBarVFull + s], 1 + 32 * kSoftmaxWarps / 2);
      mbar_init(&bar[kBarVEmpty + s], 1);
    }
    for (int h = 0; h < 8; ++h) mbar_init(&bar[kBarHand + h], 32);  // one warp's rows
    mbar_init(&bar[kBarQ], 1);
    mbar_init(&bar[kBarODone], 1);
    mbar_init(&bar[kBarDrain], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  griddep_wait();  // block lists, pairs and Q come from the preceding kernels
  // key tiles of the tile, in stream order
  const int NT = build_stream(a, m, bh, ents, reinterpret_cast<uint32_t*>(smem + L::kBm),
                              reinterpret_cast<uint32_t*>(smem + L::kCnt));
  // This work item's key tiles: all, or piece `piece` of `pieces`.
  const int i_lo = slot < 0 ? 0 : (int)((int64_t)NT * piece / a.pieces);
  const int N = slot < 0 ? NT : (int)((int64_t)NT * (piece + 1) / a.pieces) - i_lo;
  const uint32_t* units = ents + 2 * i_lo;  // units of local key tile i: units[2i], units[2i+1]
  // the build scratch in the V ring is dead; the async proxy may now write it
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Every role ends at this barrier (all 384 threads) before the tensor
  // memory is released.
  auto end_barrier = [] {
    __syncwarp();
    tc_fence_before();
    asm volatile("bar.sync 15, %0;" ::"n"(kAttnThreads) : "memory");
  };
  if (warp >= kSoftmaxWarps) {
    // warpgroup 2: producer, MMA issuer, frame means (few registers)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRegsOther));
    if (warp == kProducerWarp) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        auto load_kv = [&](int t, bool is_v) {
          const uint32_t e0 = units[2 * t], e1 = units[2 * t + 1];
          const int r0 = (int)(e0 >> 16) * 64;
          const int r1 = (int)(e1 >> 16) * 64;
          const int s = is_v ? (t % kVStages) : (t % kKStages);
          uint64_t* full = &bar[(is_v ? kBarVFull : kBarKFull) + s];
          uint8_t* dst = smem + (is_v ? L::kV : L::kK) + s * L::kTileBytes;
          const CUtensorMap* map = is_v ? &tmV : &tmK;
          mbar_arrive_expect_tx(full, L::kTileBytes);
          for (int c = 0; c < L::kChunks; ++c) {
            tma_load_3d(dst + c * L::kChunkBytes, map, full, c * 64, r0, bh);
            tma_load_3d(dst + c * L::kChunkBytes + 8192, map, full, c * 64, r1, bh);
          }
        };
        if (N > 0) {
          // the tile's two 64-row halves (a half with no query block reads past
          // the chunk's rows: zero fill)
          const int q0 = tile_row(a, bh, m, 0), q1 = tile_row(a, bh, m, 64);
          const int past = a.d.Fc * a.d.T_pad;
          mbar_arrive_expect_tx(&bar[kBarQ], L::kTileBytes);
          for (int c = 0; c < L::kChunks; ++c) {
            tma_load_3d(smem + L::kQ + c * L::kChunkBytes, &tmQ, &bar[kBarQ], c * 64, q0 < 0 ? past : q0, bh);
            tma_load_3d(smem + L::kQ + c * L::kChunkBytes + 8192, &tmQ, &bar[kBarQ], c * 64, q1 < 0 ? past : q1, bh);
          }
        }
        // Loads in the order the MMAs consume them: K(0), K(1), K(2), then
        // V(i), K(i + 3) for i = 0, 1, ... (PV(i) is followed by S(i + 3)). K(t)
        // goes to slot t mod 2 once S(t - 2) completed (SFull of its buffer),
        // V(t) to slot t mod 3 once PV(t - 3) completed. Each wait is for
        // exactly the barrier the next load needs, so the producer wakes when
        // that slot frees.
        int kt = 0, vt = 0;
        bool ok = true;
        while (ok && (kt < N || vt < N)) {
          if (kt < N && kt <= vt + kSBufs - 1) {
            if (kt >= kKStages)
              ok = mbar_wait(&bar[kBarSFull + (kt - kKStages) % kSBufs], ((kt - kKStages) / kSBufs) & 1,
                             abort_flag, a.err);
            if (ok) load_kv(kt++, false);
          } else {
            if (vt >= kVStages)
              ok = mbar_wait(&bar[kBarVEmpty + vt % kVStages], ((vt / kVStages) - 1) & 1, abort_flag, a.err);
            if (ok) load_kv(vt++, true);
          }
        }
        if (*abort_flag) {  // let copies in flight land before the CTA exits
          if (N > 0) mbar_wait_drain(&bar[kBarQ], 0);
          for (int t = (kt > kKStages ? kt - kKStages : 0); t < kt; ++t)
            mbar_wait_drain(&bar[kBarKFull + t % kKStages], (t / kKStages) & 1);
          for (int t = (vt > kVStages ? vt - kVStages : 0); t < vt; ++t)
            mbar_wait_drain(&bar[kBarVFull + t % kVStages], (t / kVStages) & 1);
        }
      }
    } else if (warp == kMmaWarp) {
      // ------------------------------------------------------------ MMA issuer
      // The whole warp runs the loop, so that the descriptors, addresses and
      // loop state are warp-uniform values; one elected lane (always the same
      // one) issues the MMAs and their commits.
      const uint64_t q_desc = smem_desc_sw128(smem_u32(smem + L::kQ), 16, 1024);
      const uint64_t k_desc = smem_desc_sw128(smem_u32(smem + L::kK), 16, 1024);
      const uint64_t v_desc = smem_desc_sw128(smem_u32(smem + L::kV), L::kChunkBytes, 1024);
      constexpr uint64_t kSlotDesc = (uint64_t)(L::kTileBytes >> 4);  // one ring slot
      const bool leader = elect_one();
      const int leader_lane = __ffs(__ballot_sync(0xFFFFFFFFu, leader)) - 1;
      // Only the issuing lane polls a barrier (32 lanes polling one mbarrier
      // would serialise on it); the result is broadcast to keep the loop
      // converged.
      auto wait_all = [&](uint64_t* b, uint32_t parity) {
        int r = 1;
        if (leader) r = mbar_wait(b, parity, abort_flag, a.err) ? 1 : 0;
        return __shfl_sync(0xFFFFFFFFu, r, leader_lane) != 0;
      };
      // S(j) into buffer j mod 3, after PV(j - 3) (which read P(j - 3) from
      // that buffer; tcgen05.mma executes in issue order).
      auto issue_score = [&](int j) -> bool {
        const int ks = j % kKStages, sb = j % kSBufs;
        if (!wait_all(&bar[kBarKFull + ks], (j / kKStages) & 1)) return false;
        tc_fence_after();
        if (leader) {
          issue_s<D>(tmem + kSCol + 128u * sb, q_desc, k_desc + (uint64_t)ks * kSlotDesc);
          mma_commit(&bar[kBarSFull + sb]);   // S(j) done: also frees K slot j mod 2
        }
        __syncwarp();
        return true;
      };
      bool ok = N > 0 && wait_all(&bar[kBarQ], 0);
      for (int j = 0; ok && j < kSBufs && j < N; ++j) ok = issue_score(j);
      for (int i = 0; ok && i < N; ++i) {
        const int sb = i % kSBufs;
        const int vs = i % kVStages;
        if (!wait_all(&bar[kBarVFull + vs], (i / kVStages) & 1)) break;   // V(i) and P(i)
        tc_fence_after();
        if (leader) {
          issue_pv<D>(tmem + kOCol, tmem + kSCol + 128u * sb, v_desc + (uint64_t)vs * kSlotDesc, i > 0);
          mma_commit(&bar[kBarVEmpty + vs]);     // V slot free = PV(i) done
          if (i + 1 == N) mma_commit(&bar[kBarODone]);  // O final: the epilogue's wait
        }
        __syncwarp();
        if (i + kSBufs < N) ok = issue_score(i + kSBufs);
      }
      if (leader) {
        mma_commit(&bar[kBarDrain]);
        mbar_wait_drain(&bar[kBarDrain], 0);
      }
      __syncwarp();
    } else if (a.kpool_frm) {
      // ------------------------------------------------------------ spare warps
      // Frame means of the chunk's new cache frames from their block means
      // (written by the previous launch), in the order of frame_pool_kernel:
      // sum_j count_j * mean_j / T_f. CTA i takes frames i, i + grid, ...
      const Dims& d = a.d;
      const int nfr = d.B * d.H * d.Fc;
      const int c0 = tid - (kMmaWarp + 1) * 32;
      constexpr int kSpare = kAttnThreads - (kMmaWarp + 1) * 32;
      for (int fr = blockIdx.x; fr < nfr; fr += gridDim.x) {
        const int fbh = fr / d.Fc;
        const int f = fr - fbh * d.Fc;
        const int fslot = (a.t0 + f) % a.W;
        const float* src = a.kpool_blk + ((size_t)fbh * a.W + fslot) * d.nb * D;
        float* dst = a.kpool_frm + ((size_t)fbh * a.W + fslot) * D;
        for (int c = c0; c < D; c += kSpare) {
          float sum = 0.f;
          for (int j = 0; j < d.nb; ++j) {
            const float cnt = (float)((j == d.nb - 1) ? d.tail : d.blk);
            sum += cnt * src[(size_t)j * D + c];
          }
          dst[c] = sum / (float)d.T_f;
        }
      }
    }
    end_barrier();
    if (warp == kMmaWarp) {
      tc_fence_after();
      tmem_dealloc(tmem, kTmemCols);
    }
  } else {
    // warpgroups 0 and 1: softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kRegsSoftmax));
    // ------------------------------------------------------------ softmax
    const Dims& d = a.d;
    const int quarter = warp & 3;        // TMEM lane quarter: rows 32 quarter .. + 31
    const int par = warp >> 2;           // this warp's key tiles: par, par + 2, par + 4, ...
    const int r = quarter * 32 + lane;   // query row of the tile = TMEM lane
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    const int mbit = r >> 6;             // this row's bit in a unit mask (warp-uniform)
    // epilogue exchange: (max, sum) [2 parities][128 rows]; flags [2 parities][4 quarters]
    float2* xch = reinterpret_cast<float2*>(smem + L::kRed);
    volatile int* okf = reinterpret_cast<volatile int*>(xch + 2 * 128);
    // hand-over of the reference maximum: one slot per row, written by the
    // warp of tile i and read by the warp of tile i + 1 (they alternate)
    volatile float* hand = reinterpret_cast<volatile float*>(smem + L::kHand);
    uint64_t* hs_out = &bar[kBarHand + 2 * quarter + par];        // my tiles' maxima
    uint64_t* hs_in = &bar[kBarHand + 2 * quarter + (par ^ 1)];   // the other warp's
    const float sc = a.scale_log2;
    float m_seen = -INFINITY;  // reference maximum (scaled log2 units) l_run is relative to
    float l_run = 0.f;
    int n_in = 0;              // hand-overs received
    bool ok = true;
    for (int i = par; ok && i < N; i += 2) {
      const int sb = i % kSBufs;
      ok = mbar_wait(&bar[kBarSFull + sb], (i / kSBufs) & 1, abort_flag, a.err);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t sbuf = trow + kSCol + 128u * sb;
      uint32_t s[4][32];
#pragma unroll
      for (int j = 0; j < 4; ++j) tmem_ld32(sbuf + 32u * j, s[j]);
      const uint32_t e0 = units[2 * i], e1 = units[2 * i + 1];
      const int lim0 = ((e0 >> mbit) & 1u) ? (int)((e0 >> 8) & 0xFFu) : 0;
      const int lim1 = ((e1 >> mbit) & 1u) ? (int)((e1 >> 8) & 0xFFu) : 0;
      const bool full = (lim0 == 64) && (lim1 == 64);   // warp-uniform
      tmem_wait_ld();
      if (!full) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int lim = j < 2 ? lim0 - 32 * j : lim1 - 32 * (j - 2);
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c >= lim) s[j][c] = __float_as_uint(-INFINITY);
        }
      }
      // four independent chains of 3-input maxima, one per 32 columns
      float mx[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        mx[j] = fmaxf(__uint_as_float(s[j][0]), __uint_as_float(s[j][1]));
#pragma unroll
        for (int c = 2; c < 32; c += 2) mx[j] = max3f(mx[j], __uint_as_float(s[j][c]), __uint_as_float(s[j][c + 1]));
      }
      const float mt = max3f(mx[0], mx[1], fmaxf(mx[2], mx[3])) * sc;  // -inf when nothing is valid
      // the reference maximum after tile i - 1, from the other warp
      float m_prev = -INFINITY;
      if (i > 0) {
        ok = mbar_wait(hs_in, n_in & 1, abort_flag, a.err);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) break;
        m_prev = hand[r];
        ++n_in;
      }
      // m only moves up: bring this warp's sum to m_prev, then decide tile i
      if (m_prev > m_seen) {
        l_run *= fast_exp2(m_seen - m_prev);   // 0 when m_seen = -inf (l_run is 0 then)
        m_seen = m_prev;
      }
      const bool need = mt > m_prev + kRescaleThreshold || (m_prev == -INFINITY && mt > -INFINITY);
      const float m_new = need ? mt : m_prev;
      if (i + 1 < N) {
        hand[r] = m_new;
        mbar_arrive(hs_out);
      }
      if (need) {
        l_run *= (m_prev == -INFINITY) ? 0.f : fast_exp2(m_prev - m_new);
        m_seen = m_new;
      }
      const float base = (m_new == -INFINITY) ? 0.f : m_new;
      const float2 sc2 = make_float2(sc, sc);
      const float2 nb2 = make_float2(-base, -base);
      float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
      // P = 2^(s sc - m) for the 128 columns, 32 at a time, on the MUFU.
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
        tmem_st16(sbuf + 16u * h, pk);
      }
      l_run += (acc0.x + acc0.y) + (acc1.x + acc1.y);
      if (__any_sync(0xFFFFFFFFu, need && m_prev > -INFINITY)) {
        // O holds PV(0 .. i-1) relative to m_prev: rescale the moving rows
        // once PV(i-1) completed (it frees V slot (i-1) mod 3). PV(i) waits
        // for this warp's P release below, so O is quiet meanwhile; the
        // rescale comes after the exponentials, when the scores' registers
        // are free.
        ok = mbar_wait(&bar[kBarVEmpty + (i - 1) % kVStages], ((i - 1) / kVStages) & 1, abort_flag, a.err);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) break;
        tc_fence_after();
        const float alpha = (need && m_prev > -INFINITY) ? fast_exp2(m_prev - m_new) : 1.f;
#pragma unroll 1
        for (int j = 0; j < D / 16; ++j) {
          uint32_t o[16];
          tmem_ld16(trow + kOCol + 16u * j, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st16(trow + kOCol + 16u * j, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar[kBarVFull + sb]);   // P(i) written (sb == V slot of tile i)
    }
    // ------------------------------------------------------------ epilogue
    // Both warps of a row range always get here and meet once: their sums
    // (each relative to the maximum it last saw) are merged. O is relative to
    // the reference after the last tile, the larger of the two maxima.
    bool fin = ok && (N == 0 || mbar_wait(&bar[kBarODone], 0, abort_flag, a.err));  // empty piece: no PV
    fin = __all_sync(0xFFFFFFFFu, fin);
    xch[par * 128 + r] = make_float2(m_seen, l_run);
    if (lane == 0) okf[par * 4 + quarter] = fin ? 1 : 0;
    pair_sync(quarter);
    fin = fin && okf[(par ^ 1) * 4 + quarter] != 0;
    if (fin) {
      if (N > 0) tc_fence_after();
      const float2 x0 = xch[r], x1 = xch[128 + r];  // parities 0 and 1
      const float M = fmaxf(x0.x, x1.x);
      const float w0 = (x0.x == -INFINITY) ? 0.f : fast_exp2(x0.x - M);
      const float w1 = (x1.x == -INFINITY) ? 0.f : fast_exp2(x1.x - M);
      const float l_tot = x0.y * w0 + x1.y * w1;
      // this warp writes columns [D/2 par, D/2 par + D/2)
      const uint32_t c0 = (uint32_t)(D / 2) * par;
      auto load_o = [&](int i, uint32_t (&o)[32]) {  // columns c0 + 32 i .. + 31, relative to M
        if (N == 0) {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
          return;
        }
        tmem_ld32(trow + kOCol + c0 + 32u * i, o);
        tmem_wait_ld();
      };
      if (slot >= 0) {
        // A piece of a split tile: O relative to M, M and the sum, for the merge launch.
        float* po = a.part_o + ((size_t)slot * kBM + r) * D + c0;
#pragma unroll
        for (int i = 0; i < D / 64; ++i) {
          uint32_t o[32];
          load_o(i, o);
          float4* dst = reinterpret_cast<float4*>(po + 32 * i);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                 __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
        }
        if (par == 0) reinterpret_cast<float2*>(a.part_ml)[(size_t)slot * kBM + r] = make_float2(M, l_tot);
      } else {
        const int pr = tile_row(a, bh, m, r);  // row in the padded chunk, or -1
        const int f = pr < 0 ? d.Fc : pr / d.T_pad;
        const int rr = pr < 0 ? 0 : pr - f * d.T_pad;
        const bool row_ok = (f < d.Fc) && (rr < d.T_f);
        const int bb = bh / d.H;
        const int h = bh - bb * d.H;
        const size_t n_tok = (size_t)f * d.T_f + rr;
        const float inv_l = (l_tot > 0.f) ? 1.f / l_tot : 0.f;
        uint16_t* orow = a.out + (((size_t)bb * d.Lq + n_tok) * d.H + h) * D + c0;
#pragma unroll
        for (int i = 0; i < D / 64; ++i) {
          uint32_t o[32];
          load_o(i, o);
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
        if (row_ok && par == 0 && a.lse)
          a.lse[(size_t)bh * d.Lq + n_tok] = (M + log2f(l_tot)) * 0.69314718055994531f;
      }
    }
    end_barrier();
  }
}

// Combines the pieces of the split tail tiles: per row, the maximum M of
// the pieces' running maxima, sum = sum_p l_p 2^(m_p - M), o = sum_p o_p
// 2^(m_p - M) / sum. One CTA per row of a split tile, D/4 threads (four
// columns each).
template <int D>
__global__ void __launch_bounds__(D / 4) attn_merge_kernel(const AttnArgs a) {
  griddep_wait();  // the pieces come from the attention launch
  const Dims& d = a.d;
  const int tt = blockIdx.x / kBM;      // split tile among the tail
  const int r = blockIdx.x - tt * kBM;  // row of the tile
  const int tile = a.Qf + tt;
  const int bh = tile / a.MT;
  const int m = tile - bh * a.MT;
  const int s0 = tt * a.pieces;
  const float2* ml = reinterpret_cast<const float2*>(a.part_ml);
  // One pass over the pieces, eight at a time (their loads independent of
  // one another): the running maximum M and the sums rescaled when it grows.
  float M = -INFINITY;
  float lsum = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const int c = 4 * threadIdx.x;
  for (int p0 = 0; p0 < a.pieces; p0 += 8) {
    float2 e[8];
    float4 o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const size_t row = (size_t)(s0 + p0 + j) * kBM + r;
      const bool in = p0 + j < a.pieces;
      e[j] = in ? ml[row] : make_float2(-INFINITY, 0.f);
      o[j] = in ? *reinterpret_cast<const float4*>(a.part_o + row * D + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float bm = M;
#pragma unroll
    for (int j = 0; j < 8; ++j) bm = fmaxf(bm, e[j].x);
    if (bm > M) {
      const float sc = (M == -INFINITY) ? 0.f : exp2f(M - bm);
      lsum *= sc;
      acc.x *= sc;
      acc.y *= sc;
      acc.z *= sc;
      acc.w *= sc;
      M = bm;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float w = (e[j].x == -INFINITY) ? 0.f : exp2f(e[j].x - M);
      lsum += w * e[j].y;
      acc.x += w * o[j].x;
      acc.y += w * o[j].y;
      acc.z += w * o[j].z;
      acc.w += w * o[j].w;
    }
  }
  const int pr = tile_row(a, bh, m, r);
  if (pr < 0) return;
  const int f = pr / d.T_pad;
  const int rr = pr - f * d.T_pad;
  if (f >= d.Fc || rr >= d.T_f) return;
  const int bb = bh / d.H;
  const int h = bh - bb * d.H;
  const size_t n_tok = (size_t)f * d.T_f + rr;
  const float inv = (lsum > 0.f) ? 1.f / lsum : 0.f;
  uint2 pk;
  pk.x = cvt_bf16x2(acc.x * inv, acc.y * inv);
  pk.y = cvt_bf16x2(acc.z * inv, acc.w * inv);
  *reinterpret_cast<uint2*>(a.out + (((size_t)bb * d.Lq + n_tok) * d.H + h) * D + c) = pk;
  if (threadIdx.x == 0 && a.lse) a.lse[(size_t)bh * d.Lq + n_tok] = (M + log2f(lsum)) * 0.69314718055994531f;
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
bool make_map_2d(CUtensorMap* map, const void* base, bool fp32, uint64_t d0, uint64_t d1,
                 uint64_t row_bytes, uint32_t box0, uint32_t box1) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {d0, d1};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box0, box1};
  cuuint32_t es[2] = {1, 1};
  const CUresult r = enc(map, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                         const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_map(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
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
                                      const CUtensorMap& mv, cudaStream_t stream, bool dependent) {
  using L = AttnSmem<D>;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       L::kAlloc);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  const int tiles = a.MT * a.d.B * a.d.H;
  dim3 grid(a.Qf + (tiles - a.Qf) * a.pieces);
  e = launch_kernel(attn_fwd_kernel<D>, grid, dim3(kAttnThreads), L::kAlloc, stream, dependent, mq, mk, mv, a);
  if (e != cudaSuccess || a.Qf == tiles) return e;
  // the merge always follows the attention launch
  return launch_kernel(attn_merge_kernel<D>, dim3((tiles - a.Qf) * kBM), dim3(D / 4), 0, stream, true, a);
}

cudaError_t launch_attention(const AttnArgs& a, const void* q_rot, const void* cache_k,
                             const void* cache_v, cudaStream_t stream, const char** why, bool dependent) {
  const Dims& d = a.d;
  CUtensorMap mq, mk, mv;
  const uint64_t bh = (uint64_t)d.B * d.H;
  if (!make_map(&mq, q_rot, d.D, (uint64_t)d.Fc * d.T_pad, bh, 64) ||
      !make_map(&mk, cache_k, d.D, (uint64_t)a.W * d.T_pad, bh, 64) ||
      !make_map(&mv, cache_v, d.D, (uint64_t)a.W * d.T_pad, bh, 64)) {
    *why = "cuTensorMapEncodeTiled failed (driver entry point or tensor shape)";
    return cudaErrorInvalidValue;
  }
  return d.D == 128 ? launch_attention_d<128>(a, mq, mk, mv, stream, dependent)
                    : launch_attention_d<64>(a, mq, mk, mv, stream, dependent);
}

}  // namespace cva
