// QKV projection fused with Causal-RoPE, the cache append and block pooling.
//
// "Accelerating Video Generation Inference with Sequential-Parallel 3D
// Positional Encoding Using a Global Time Index", section 2C (operator
// fusion): the QKV projection and the Causal-RoPE computation run as one
// kernel; section 2B: a token of local frame f of a chunk starting at
// global frame t0 is rotated with temporal coordinate t0 + f.
//
// y = x W^T for the chunk's tokens (x [B, Lq, C], W [3 H D, C]: rows q
// heads, then k heads, then v heads; no bias), on the tensor cores:
// tcgen05.mma kind::f16, bf16 operands staged by TMA (128-byte swizzle, no
// multicast) through a 4-stage ring, fp32 accumulators in tensor memory.
// One CTA computes a 128 x 256 tile of y. Its 128 rows are PADDED token
// rows (frames padded to whole blocks, the attention's layout): two 64-row
// halves, each loaded from the token rows of one 64-row piece of a frame,
// so a tile never needs a gather beyond two boxes per k-step. Rows past a
// frame's last token read whatever follows and are written as zeros.
//
// Epilogue (4 warps, thread = row): the accumulator row is read 32 columns
// at a time; q and k columns are rotated in fp32 with the precomputed
// cos/sin tables and rounded once to bf16; q goes to Q_rot
// [B][H][Fc*T_pad][D], k and v to the cache slot of their frame (t mod W).
// Block means of the stored bf16 q and k values (per query block / cache
// block) are reduced across the rows of a block in a fixed order (warp
// shuffles, then the warps of the block in order), as the attention's
// selection step needs them.
//
// Persistent: one CTA per SM walks its tiles (grouped order for L2 reuse);
// the accumulator is double-buffered in tensor memory (2 x 256 columns), so
// the MMAs of the next tile run while the epilogue rotates and stores the
// previous one. The epilogue warps also stage the cos/sin rows of the chunk
// in shared memory before the first tile.
//
// Roles (192 threads): warps 0-3 epilogue, warp 4 TMA producer (one lane),
// warp 5 MMA issuer (one lane; also allocates the 512 TMEM columns). Every
// wait is bounded (4 s, then CVA_DEV_TIMEOUT and every role leaves).
#include <cudaTypedefs.h>

#include "kernels.cuh"

namespace cva {

constexpr int kQkvBM = 128;
constexpr int kQkvBN = 256;
constexpr int kQkvBK = 64;       // one 128-byte swizzle row of bf16
constexpr int kQkvStages = 4;
constexpr int kQkvEpiWarps = 8;   // two per TMEM lane quarter, each half of the columns
constexpr int kQkvThreads = 32 * kQkvEpiWarps + 64;
constexpr int kQkvProducerWarp = kQkvEpiWarps;
constexpr int kQkvMmaWarp = kQkvEpiWarps + 1;
constexpr int kQkvGroupM = 8;

struct QkvSmem {
  static constexpr int kABytes = kQkvBM * kQkvBK * 2;  // 16 KB: two 64-row boxes
  static constexpr int kBBytes = kQkvBN * kQkvBK * 2;  // 32 KB
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kA = 0;                         // stage s at + s * kStageBytes
  static constexpr int kB = kABytes;
  static constexpr int kRed = kQkvStages * kStageBytes;  // [2 groups][2][4 warps][32] column sums
  static constexpr int kTab = kRed + 2 * 2 * 4 * 32 * 4;   // cos/sin tables of the chunk
  static constexpr int kTabFloats = 7168;
  static constexpr int kBar = kTab + kTabFloats * 4;
  static constexpr int kMisc = kBar + 16 * 8;
  static constexpr int kBytes = kMisc + 64;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 232448, "shared memory of one CTA");
};

// Barriers: stage s full / empty; accumulator buffer u full (MMAs done) /
// empty (epilogue done reading it).
constexpr int kQBarFull = 0, kQBarEmpty = kQkvStages, kQBarAccFull = 2 * kQkvStages,
              kQBarAccEmpty = 2 * kQkvStages + 2;

__device__ __forceinline__ void qkv_epi_sync() {  // all epilogue warps
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kQkvEpiWarps) : "memory");
}
__device__ __forceinline__ void qkv_group_sync(int g) {  // the 4 warps of column half g
  asm volatile("bar.sync %0, 128;" ::"r"(2 + g) : "memory");
}

__global__ void __launch_bounds__(kQkvThreads, 1)
    qkv_rope_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                    const QkvArgs a) {
  griddep_launch_dependents();
  using L = QkvSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const Dims& d = a.d;
  // Persistent: CTA c takes tiles c, c + gridDim.x, ... Tile order: per
  // batch, groups of kQkvGroupM row tiles; inside a group the column tile is
  // the slower index, so the CTAs that run together share a few weight
  // tiles and a few row tiles (both stay in L2).
  const int ntiles = d.B * a.MT * a.NT;
  auto decode = [&](int id, int& b, int& mt, int& nt) {
    b = id / (a.MT * a.NT);
    id -= b * (a.MT * a.NT);
    const int g = id / (kQkvGroupM * a.NT);
    const int r0 = id - g * (kQkvGroupM * a.NT);
    const int gm = min(kQkvGroupM, a.MT - g * kQkvGroupM);
    nt = r0 / gm;
    mt = g * kQkvGroupM + (r0 - nt * gm);
  };
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  const int KT = a.C / kQkvBK;

  if (tid == 0) {
    for (int s = 0; s < kQkvStages; ++s) {
      mbar_init(&bar[kQBarFull + s], 1);
      mbar_init(&bar[kQBarEmpty + s], 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(&bar[kQBarAccFull + u], 1);
      mbar_init(&bar[kQBarAccEmpty + u], 32 * kQkvEpiWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kQkvMmaWarp) {
    tmem_alloc(tmem_slot, 2 * kQkvBN);  // two accumulator buffers
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kQkvProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(&tmW);
      int issued = 0;  // k-steps over all of this CTA's tiles: stage issued % S
      bool ok = true;
      for (int id = blockIdx.x; ok && id < ntiles; id += gridDim.x) {
        int b, mt, nt;
        decode(id, b, mt, nt);
        // token row of each 64-row half of the tile (Lq: past the end, zero-filled)
        int tok[2];
        for (int h = 0; h < 2; ++h) {
          const int pr = mt * kQkvBM + 64 * h;
          const int f = pr / d.T_pad;
          tok[h] = (f < d.Fc) ? f * d.T_f + (pr - f * d.T_pad) : d.Lq;
        }
        for (int k = 0; k < KT; ++k) {
          const int s = issued % kQkvStages;
          if (issued >= kQkvStages &&
              !mbar_wait(&bar[kQBarEmpty + s], ((issued / kQkvStages) - 1) & 1, abort_flag, a.err)) {
            ok = false;
            break;
          }
          ++issued;
          uint8_t* st = smem + s * L::kStageBytes;
          mbar_arrive_expect_tx(&bar[kQBarFull + s], L::kStageBytes);
          tma_load_3d(st + L::kA, &tmX, &bar[kQBarFull + s], k * kQkvBK, tok[0], b);
          tma_load_3d(st + L::kA + 8192, &tmX, &bar[kQBarFull + s], k * kQkvBK, tok[1], b);
          tma_load_3d(st + L::kB, &tmW, &bar[kQBarFull + s], k * kQkvBK, nt * kQkvBN, 0);
        }
      }
      if (*abort_flag) {  // let copies in flight land before the CTA exits
        for (int k = (issued > kQkvStages ? issued - kQkvStages : 0); k < issued; ++k) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&bar[kQBarFull + k % kQkvStages], (k / kQkvStages) & 1))
            if (globaltimer_ns() - t0 > 200000000ull) break;
        }
      }
    }
  } else if (warp == kQkvMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kId = idesc_bf16_f32(kQkvBM, kQkvBN, 0, 0);  // both K-major
      bool ok = true;
      int used = 0;  // k-steps consumed over all tiles
      for (int id = blockIdx.x, lt = 0; ok && id < ntiles; id += gridDim.x, ++lt) {
        const int u = lt & 1;  // accumulator buffer of this tile
        // the epilogue must have read the tile that used buffer u before
        if (lt >= 2 && !mbar_wait(&bar[kQBarAccEmpty + u], ((lt >> 1) - 1) & 1, abort_flag, a.err)) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(u * kQkvBN);
        for (int k = 0; k < KT; ++k, ++used) {
          const int s = used % kQkvStages;
          ok = mbar_wait(&bar[kQBarFull + s], (used / kQkvStages) & 1, abort_flag, a.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * L::kStageBytes + L::kA);
          const uint32_t b_addr = smem_u32(smem + s * L::kStageBytes + L::kB);
#pragma unroll
          for (int kk = 0; kk < kQkvBK / 16; ++kk)
            mma_ss(acc, smem_desc_sw128(a_addr + 32u * kk, 16, 1024), smem_desc_sw128(b_addr + 32u * kk, 16, 1024),
                   kId, (k > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bar[kQBarEmpty + s]);
        }
        if (ok) mma_commit(&bar[kQBarAccFull + u]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;        // TMEM lane quarter
    const int grp = warp >> 2;           // column half: chunks 4 grp .. 4 grp + 3
    const int r = quarter * 32 + lane;   // row of the tile = TMEM lane
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    volatile int* okw = reinterpret_cast<volatile int*>(smem + L::kMisc + 16);  // [8]
    // While the MMAs run: copy the cos/sin rows the chunk needs into shared
    // memory: [cos_t, sin_t] of frames t0 .. t0+Fc-1, then [cos_h, sin_h]
    // (Fh rows), then [cos_w, sin_w] (Fw rows).
    const int nt_f = d.Fc * a.tab.pt, nh_f = d.Fh * a.tab.ph, nw_f = d.Fw * a.tab.pw;
    const bool stab = 2 * (nt_f + nh_f + nw_f) <= L::kTabFloats;  // uniform
    float* tb = reinterpret_cast<float*>(smem + L::kTab);
    if (stab) {
      const float* src_t = a.tab.cos_t + (size_t)a.t0 * a.tab.pt;
      const float* src_ts = a.tab.sin_t + (size_t)a.t0 * a.tab.pt;
      constexpr int kN = 32 * kQkvEpiWarps;
      for (int i = tid; i < nt_f; i += kN) { tb[i] = src_t[i]; tb[nt_f + i] = src_ts[i]; }
      float* th = tb + 2 * nt_f;
      for (int i = tid; i < nh_f; i += kN) { th[i] = a.tab.cos_h[i]; th[nh_f + i] = a.tab.sin_h[i]; }
      float* tw = th + 2 * nh_f;
      for (int i = tid; i < nw_f; i += kN) { tw[i] = a.tab.cos_w[i]; tw[nw_f + i] = a.tab.sin_w[i]; }
    }
    qkv_epi_sync();
    for (int id = blockIdx.x, lt = 0; id < ntiles; id += gridDim.x, ++lt) {
      int b, mt, nt;
      decode(id, b, mt, nt);
      const int u = lt & 1;  // accumulator buffer of this tile
      bool ok = mbar_wait(&bar[kQBarAccFull + u], (lt >> 1) & 1, abort_flag, a.err);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (lane == 0) okw[warp] = ok ? 1 : 0;
      qkv_epi_sync();  // the epilogue warps take the same path through the barriers below
      ok = true;
#pragma unroll
      for (int w = 0; w < kQkvEpiWarps; ++w) ok = ok && okw[w] != 0;
      qkv_epi_sync();  // okw is rewritten for the next tile
      if (!ok) break;
      tc_fence_after();
      const uint32_t tacc = trow + (uint32_t)(u * kQkvBN);
      const int pr = mt * kQkvBM + r;  // padded row in the chunk
      const int f = pr / d.T_pad;
      const int rr = pr - f * d.T_pad;
      const bool in_chunk = f < d.Fc;
      const bool valid = in_chunk && rr < d.T_f;
      const int t = a.t0 + f;
      const int slot = t % a.W;
      const int hh = rr / d.Fw;
      const int ww = rr - hh * d.Fw;
      // table row offsets of this row (position 0 for rows that are not
      // tokens); the staged time table starts at frame t0
      const size_t t_off = valid ? (size_t)(stab ? f : t) * a.tab.pt : 0;
      const size_t h_off = valid ? (size_t)hh * a.tab.ph : 0;
      const size_t w_off = valid ? (size_t)ww * a.tab.pw : 0;
      const float* tct = stab ? tb : a.tab.cos_t;
      const float* tst = stab ? tb + nt_f : a.tab.sin_t;
      const float* tch = stab ? tb + 2 * nt_f : a.tab.cos_h;
      const float* tsh = stab ? tb + 2 * nt_f + nh_f : a.tab.sin_h;
      const float* tcw = stab ? tb + 2 * nt_f + 2 * nh_f : a.tab.cos_w;
      const float* tsw = stab ? tb + 2 * nt_f + 2 * nh_f + nw_f : a.tab.sin_w;
      const int j = rr / d.blk;                  // block of the frame
      const int jb = f * d.nb + j;               // query block of the chunk
      const float vcnt = (float)((j == d.nb - 1) ? d.tail : d.blk);
      const int wpb = d.blk / 32;                // warps per block
      const int w0 = (quarter / wpb) * wpb;      // first lane quarter of this row's block
      const int HD = d.H * d.D;
      float* red = reinterpret_cast<float*>(smem + L::kRed) + grp * 2 * 128;
      for (int cc = 4 * grp; cc < 4 * grp + 4; ++cc) {
        const int c = nt * kQkvBN + 32 * cc;
        if (c >= 3 * HD) break;                  // uniform: the projection has 3HD outputs
        const int which = c / HD;                // 0 q, 1 k, 2 v
        const int rem = c - which * HD;
        const int head = rem / d.D;
        const int d0 = rem - head * d.D;
        uint32_t o[32];
        tmem_ld32(tacc + 32u * cc, o);
        tmem_wait_ld();
        uint32_t pk[16];
        if (which < 2) {
          // cos/sin of the chunk's 16 pairs: all loads issued before any use
          // (pad rows use position 0; their output is zero anyway)
          float cs[16], sn[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int p = (d0 >> 1) + i;       // warp-uniform
            const float* ct;
            const float* stb;
            size_t off;
            if (p < a.tab.pt) {
              ct = tct; stb = tst; off = t_off + p;
            } else if (p < a.tab.pt + a.tab.ph) {
              ct = tch; stb = tsh; off = h_off + (p - a.tab.pt);
            } else {
              ct = tcw; stb = tsw; off = w_off + (p - a.tab.pt - a.tab.ph);
            }
            cs[i] = ct[off];
            sn[i] = stb[off];
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float y0 = __uint_as_float(o[2 * i]), y1 = __uint_as_float(o[2 * i + 1]);
            pk[i] = valid ? cvt_bf16x2(y0 * cs[i] - y1 * sn[i], y0 * sn[i] + y1 * cs[i]) : 0u;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = valid ? cvt_bf16x2(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1])) : 0u;
        }
        if (in_chunk) {
          const size_t bh = (size_t)b * d.H + head;
          uint16_t* dst;
          if (which == 0) dst = a.q_rot + (bh * (size_t)(d.Fc * d.T_pad) + pr) * d.D + d0;
          else dst = (which == 1 ? a.k_cache : a.v_cache) + ((bh * a.W + slot) * d.T_pad + rr) * d.D + d0;
          uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
          for (int v = 0; v < 4; ++v) d4[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
        float* pool = which == 0 ? a.qpool : (which == 1 ? a.kpool_blk : nullptr);
        if (pool) {                              // uniform
          // column sums of the stored bf16 values over this warp's rows:
          // reduce-scatter, lane i ends with column d0 + i
          float v[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            v[2 * i] = bf16_lo(pk[i]);
            v[2 * i + 1] = bf16_hi(pk[i]);
          }
#pragma unroll
          for (int ofs = 16; ofs >= 1; ofs >>= 1) {
            const bool upper = (lane & ofs) != 0;
#pragma unroll
            for (int i = 0; i < ofs; ++i) {
              const float send = upper ? v[i] : v[i + ofs];
              const float keep = upper ? v[i + ofs] : v[i];
              v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, ofs);
            }
          }
          float* rb = red + (cc & 1) * 128;
          rb[quarter * 32 + lane] = v[0];
          qkv_group_sync(grp);
          const int prb = mt * kQkvBM + w0 * 32;   // first row of the block
          if (quarter == w0 && prb / d.T_pad < d.Fc) {
            float s = 0.f;
            for (int w = 0; w < wpb; ++w) s += rb[(w0 + w) * 32 + lane];
            const size_t bh = (size_t)b * d.H + head;
            if (which == 0) pool[(bh * d.NQB + jb) * d.D + d0 + lane] = s / vcnt;
            else pool[((bh * a.W + slot) * d.nb + j) * d.D + d0 + lane] = s / vcnt;
          }
        }
      }
      // buffer u is read: the MMAs of the tile after next may overwrite it
      tc_fence_before();
      mbar_arrive(&bar[kQBarAccEmpty + u]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kQkvMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kQkvBN);
  }
}

cudaError_t launch_qkv_rope(const QkvArgs& a, const void* x, const void* w, cudaStream_t stream,
                            const char** why) {
  const Dims& d = a.d;
  CUtensorMap mx, mw;
  if (!make_map(&mx, x, (uint64_t)a.C, (uint64_t)d.Lq, (uint64_t)d.B, 64) ||
      !make_map(&mw, w, (uint64_t)a.C, (uint64_t)3 * d.H * d.D, 1, kQkvBN)) {
    *why = "cuTensorMapEncodeTiled failed (driver entry point or tensor shape)";
    return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(qkv_rope_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       QkvSmem::kAlloc);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    nsm = 148;
  const int ntiles = a.NT * a.MT * d.B;
  dim3 grid(ntiles < nsm ? ntiles : nsm);  // persistent: one CTA per SM
  qkv_rope_kernel<<<grid, kQkvThreads, QkvSmem::kAlloc, stream>>>(mx, mw, a);
  return cudaGetLastError();
}

}  // namespace cva
