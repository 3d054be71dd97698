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
// One CTA handles one (batch*head, frame, block) of up to three tensors
// (Q, K, V) in a single pass over HBM. Each thread owns 8 consecutive
// elements (one 16-byte vector) of a row, so a warp reads and writes whole
// rows. rope_pool_tma_kernel (below) stages the block's rows and its rows of
// the per-position (cos, sin) table in shared memory through TMA;
// rope_pool_kernel, for tables without the per-position expansion, loads a
// batch of rows into registers and looks every pair up in the per-axis
// tables. The job properties (which tensors are rotated or pooled) are
// template parameters, so the per-row work is the loads, the rotation, the
// pooling sums and the stores. Block sums are reduced in a fixed order from
// the bf16 values actually stored (deterministic). Frame means of the block
// means are a separate step (frame_pool_kernel, or the attention kernel's
// spare warps in the fused chunk call).
#include "kernels.cuh"

namespace cva {

// Compile-time job properties: rotation and block pooling of jobs 0 and 1
// (job 2, when present, is a plain copy).
enum : int { kRot0 = 1, kRot1 = 2, kPool0 = 4, kPool1 = 8 };

// Addressing of one job in a block: the thread's vector in its first row
// and the row stride (elements).
struct JobRows {
  const uint16_t* src;
  uint16_t* dst;
  int sstride, dstride;
  bool tok_dst;
};

template <int D>
__device__ __forceinline__ JobRows job_rows(const StreamJob& job, const Dims& d, int b, int h, int bh,
                                            int f, int slot, int W, int row, int col) {
  JobRows r;
  if (job.src_layout == kTokenMajor) {
    r.src = job.src + (((size_t)b * d.Lq + (size_t)f * d.T_f + row) * d.H + h) * D + col;
    r.sstride = d.H * D;
  } else {
    r.src = job.src + ((size_t)bh * d.Fc * d.T_pad + (size_t)f * d.T_pad + row) * D + col;
    r.sstride = D;
  }
  r.dst = nullptr;
  r.dstride = D;
  r.tok_dst = false;
  if (job.dst) {
    if (job.dst_layout == kTokenMajor) {
      r.dst = job.dst + (((size_t)b * d.Lq + (size_t)f * d.T_f + row) * d.H + h) * D + col;
      r.dstride = d.H * D;
      r.tok_dst = true;
    } else if (job.dst_layout == kHeadMajor) {
      r.dst = job.dst + ((size_t)bh * d.Fc * d.T_pad + (size_t)f * d.T_pad + row) * D + col;
    } else {
      r.dst = job.dst + (((size_t)bh * W + slot) * d.T_pad + row) * D + col;
    }
  }
  return r;
}

// Rotation of 4 adjacent pairs packed as bf16: (x0, x1) -> (x0 c - x1 s, x0 s + x1 c),
// as (x0, x0) * (c, s) followed by (x1, x1) * (-s, c) + that, on f32x2 pairs.
__device__ __forceinline__ uint4 rotate4(uint4 v, const float (&c)[4], const float (&s)[4]) {
  const uint32_t in[4] = {v.x, v.y, v.z, v.w};
  uint32_t out[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float x0 = bf16_lo(in[i]);
    const float x1 = bf16_hi(in[i]);
    const float2 t = fmul2(make_float2(x0, x0), make_float2(c[i], s[i]));
    const float2 y = ffma2(make_float2(x1, x1), make_float2(-s[i], c[i]), t);
    out[i] = pack_bf16(y.x, y.y);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

__device__ __forceinline__ void pool_add(float (&acc)[8], uint4 y) {
  const uint32_t in[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 r = fadd2(make_float2(acc[2 * i], acc[2 * i + 1]), make_float2(bf16_lo(in[i]), bf16_hi(in[i])));
    acc[2 * i] = r.x;
    acc[2 * i + 1] = r.y;
  }
}

// The CTA's column sums of one job: the lanes of a warp that share a column
// group add up through shuffles, then warp w's sums go to red[w][D] (fixed
// order). The caller synchronises before reading red.
template <int D>
__device__ __forceinline__ void warp_col_sums(const float (&acc)[8], float* red, int tid) {
  constexpr int kCG = D / 8;
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = acc[i];
#pragma unroll
  for (int o = kCG; o < 32; o <<= 1)
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] += __shfl_xor_sync(0xFFFFFFFFu, v[i], o);
  const int lane = tid & 31;
  if (lane < kCG) {
    float4* dst = reinterpret_cast<float4*>(red + (tid >> 5) * D + lane * 8);
    dst[0] = make_float4(v[0], v[1], v[2], v[3]);
    dst[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

// NJ jobs (1..3) with the properties FL; rows of a block in batches of ROWS;
// at least MINB CTAs per SM.
template <int D, int NJ, int FL, int ROWS, int MINB>
__global__ void __launch_bounds__(256, MINB) rope_pool_kernel(RopePoolArgs a) {
  griddep_launch_dependents();
  constexpr int kCG = D / 8;         // column groups (16-byte vectors) per row
  constexpr int kRP = 256 / kCG;     // rows per pass
  constexpr int kPass = ROWS / kRP;  // passes per batch
  constexpr bool kRot[3] = {(FL & kRot0) != 0, (FL & kRot1) != 0, false};
  constexpr bool kPool[3] = {(FL & kPool0) != 0, (FL & kPool1) != 0, false};
  constexpr bool kAnyRot = (FL & (kRot0 | kRot1)) != 0;
  static_assert(NJ >= 1 && NJ <= 3 && kPass >= 1, "bad configuration");
  __shared__ __align__(16) float red[8][D];

  const Dims& d = a.d;
  const int f = blockIdx.x / d.nb;
  const int j = blockIdx.x - f * d.nb;
  const int bh = blockIdx.y;
  const int b = bh / d.H;
  const int h = bh - b * d.H;
  const int tid = threadIdx.x;
  const int cgi = tid % kCG;
  const int rg = tid / kCG;
  const int valid = (j == d.nb - 1) ? d.tail : d.blk;
  const int t = a.t0 + f;
  const int slot = t % a.W;
  const int row0 = j * d.blk;

  JobRows jr[NJ];
#pragma unroll
  for (int jb = 0; jb < NJ; ++jb) jr[jb] = job_rows<D>(a.job[jb], d, b, h, bh, f, slot, a.W, row0 + rg, cgi * 8);

  // This thread's 4 pairs: axis (0 t, 1 h, 2 w) and table column.
  int axis[4], col[4];
  float ct[4], st[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int p = cgi * 4 + i;
    if (p < a.tab.pt) {
      axis[i] = 0; col[i] = p;
    } else if (p < a.tab.pt + a.tab.ph) {
      axis[i] = 1; col[i] = p - a.tab.pt;
    } else {
      axis[i] = 2; col[i] = p - a.tab.pt - a.tab.ph;
    }
  }
  const float* cs_tok = a.tab.cs_tok;  // per-position table, or nullptr (per-axis lookups)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    ct[i] = 1.f;
    st[i] = 0.f;
    if (kAnyRot && axis[i] == 0) {
      ct[i] = __ldg(a.tab.cos_t + (size_t)t * a.tab.pt + col[i]);
      st[i] = __ldg(a.tab.sin_t + (size_t)t * a.tab.pt + col[i]);
    }
  }

  float acc[2][8];
#pragma unroll
  for (int jb = 0; jb < 2; ++jb)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[jb][i] = 0.f;
  int hh = 0, ww = 0;
  if (kAnyRot) {
    hh = (row0 + rg) / d.Fw;
    ww = row0 + rg - hh * d.Fw;
  }

  for (int g = 0; g < d.blk; g += ROWS) {
    uint4 x[NJ][kPass];
    float4 cs4[kPass][2];  // (c0, s0, c1, s1), (c2, s2, c3, s3) of this thread's pairs
#pragma unroll
    for (int p = 0; p < kPass; ++p) {
      cs4[p][0] = make_float4(1.f, 0.f, 1.f, 0.f);
      cs4[p][1] = make_float4(1.f, 0.f, 1.f, 0.f);
    }
    const bool full = g + ROWS <= valid;
#pragma unroll
    for (int p = 0; p < kPass; ++p) {
      const bool live = full || g + p * kRP + rg < valid;
#pragma unroll
      for (int jb = 0; jb < NJ; ++jb) {
        x[jb][p] = make_uint4(0u, 0u, 0u, 0u);
        if (live) x[jb][p] = __ldcs(reinterpret_cast<const uint4*>(jr[jb].src + (size_t)(g + p * kRP) * jr[jb].sstride));
      }
    }
    if (kAnyRot && cs_tok && cgi * 4 + 3 >= a.tab.pt) {  // threads with a spatial pair
      int h2 = hh, w2 = ww;
#pragma unroll
      for (int p = 0; p < kPass; ++p) {
        const bool live = full || g + p * kRP + rg < valid;
        if (live) {
          const float4* e = reinterpret_cast<const float4*>(cs_tok + ((size_t)(h2 * a.tab.tab_w + w2) * (D / 2) + 4 * cgi) * 2);
          cs4[p][0] = __ldg(e);
          cs4[p][1] = __ldg(e + 1);
        }
        w2 += kRP;
        while (w2 >= d.Fw) {
          w2 -= d.Fw;
          ++h2;
        }
      }
    }
#pragma unroll
    for (int p = 0; p < kPass; ++p) {
      const bool live = full || g + p * kRP + rg < valid;
      float c[4], s[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        c[i] = kAnyRot ? ct[i] : 1.f;
        s[i] = kAnyRot ? st[i] : 0.f;
      }
      if (kAnyRot && cs_tok) {
        const float e[8] = {cs4[p][0].x, cs4[p][0].y, cs4[p][0].z, cs4[p][0].w,
                            cs4[p][1].x, cs4[p][1].y, cs4[p][1].z, cs4[p][1].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (axis[i] != 0) {
            c[i] = e[2 * i];
            s[i] = e[2 * i + 1];
          }
        }
      } else if (kAnyRot && live) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (axis[i] == 1) {
            c[i] = __ldg(a.tab.cos_h + hh * a.tab.ph + col[i]);
            s[i] = __ldg(a.tab.sin_h + hh * a.tab.ph + col[i]);
          } else if (axis[i] == 2) {
            c[i] = __ldg(a.tab.cos_w + ww * a.tab.pw + col[i]);
            s[i] = __ldg(a.tab.sin_w + ww * a.tab.pw + col[i]);
          }
        }
      }
#pragma unroll
      for (int jb = 0; jb < NJ; ++jb) {
        uint4 y = x[jb][p];
        if (kRot[jb] && live) y = rotate4(y, c, s);
        if (kPool[jb]) pool_add(acc[jb], y);
        if (jr[jb].dst && (live || !jr[jb].tok_dst))
          *reinterpret_cast<uint4*>(jr[jb].dst + (size_t)(g + p * kRP) * jr[jb].dstride) = y;
      }
      if (kAnyRot) {
        ww += kRP;
        while (ww >= d.Fw) {
          ww -= d.Fw;
          ++hh;
        }
      }
    }
  }

  // block means, reduced over the rows in a fixed order
#pragma unroll
  for (int jb = 0; jb < 2; ++jb) {
    if (!kPool[jb] || jb >= NJ) continue;
    warp_col_sums<D>(acc[jb], &red[0][0], tid);
    __syncthreads();
    if (tid < D) {
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) sum += red[w][tid];
      const StreamJob& job = a.job[jb];
      size_t off;
      if (job.pool_layout == kPoolChunk) {
        off = ((size_t)bh * d.NQB + (size_t)f * d.nb + j) * D + tid;
      } else {
        off = (((size_t)bh * a.W + slot) * d.nb + j) * D + tid;
      }
      job.pool[off] = sum / (float)valid;
    }
    __syncthreads();
  }
}

// ---- the staged variant: tiles brought in by TMA ---------------------------
//
// The block's rows go in groups of 32 through two shared-memory buffers: one
// thread issues, per group, one 2D tiled TMA load per tensor (32 rows x D
// columns of the token-major or head-major source) and one of the
// per-position (cos, sin) table (its spatial columns), all completing on the
// buffer's mbarrier. The first two groups are in flight together; the CTA
// works on one while the other lands, without holding them in registers.
template <int D>
struct RopeTma {
  static constexpr int kRows = 32;                        // rows per group
  static constexpr int kPt = D / 2 - 2 * ((D / 2) / 3);  // temporal pairs
  static constexpr int kTabX = 8 * (kPt / 4);            // first float of the first group with a spatial pair
  static constexpr int kTabW = D - kTabX;                 // table floats per row in the tile
  static constexpr int kTile = kRows * D * 2;             // bytes of one tensor's tile
  static constexpr int kTab = kRows * kTabW * 4;          // bytes of the table tile
  static_assert((kTabX * 4) % 16 == 0 && (kTabW * 4) % 16 == 0, "TMA alignment");
  __host__ __device__ static constexpr int buf_bytes(int nj, bool tab) { return nj * kTile + (tab ? kTab : 0); }
};

template <int D, int NJ, int FL, bool TOK>
__global__ void __launch_bounds__(256, 3)
    rope_pool_tma_kernel(const __grid_constant__ CUtensorMap m0, const __grid_constant__ CUtensorMap m1,
                         const __grid_constant__ CUtensorMap m2, const __grid_constant__ CUtensorMap mt,
                         RopePoolArgs a) {
  griddep_launch_dependents();
  using L = RopeTma<D>;
  constexpr int kCG = D / 8;
  constexpr int kRP = 256 / kCG;
  constexpr int kPass = L::kRows / kRP;
  constexpr bool kRot[3] = {(FL & kRot0) != 0, (FL & kRot1) != 0, false};
  constexpr bool kPool[3] = {(FL & kPool0) != 0, (FL & kPool1) != 0, false};
  constexpr bool kAnyRot = (FL & (kRot0 | kRot1)) != 0;
  constexpr bool kTab = TOK && kAnyRot;
  constexpr int kBuf = L::buf_bytes(NJ, kTab);
  static_assert(!kAnyRot || TOK, "rotation needs the per-position table");
  static_assert(kPass >= 1, "bad configuration");
  extern __shared__ __align__(128) uint8_t rp_smem[];
  // buffer q: NJ tiles [32][D] bf16, then the table tile [32][kTabW] fp32
  uint64_t* bar = reinterpret_cast<uint64_t*>(rp_smem + 2 * kBuf);        // [2]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 2);
  float* red = reinterpret_cast<float*>(rp_smem);                          // [8][D], after the last group

  const Dims& d = a.d;
  const int f = blockIdx.x / d.nb;
  const int j = blockIdx.x - f * d.nb;
  const int bh = blockIdx.y;
  const int b = bh / d.H;
  const int h = bh - b * d.H;
  const int tid = threadIdx.x;
  const int cgi = tid % kCG;
  const int rg = tid / kCG;
  const int valid = (j == d.nb - 1) ? d.tail : d.blk;
  const int t = a.t0 + f;
  const int slot = t % a.W;
  const int row0 = j * d.blk;
  const int ngroups = d.blk / L::kRows;
  const CUtensorMap* maps[3] = {&m0, &m1, &m2};

  // source coordinates of row 0 of the block
  int sx[NJ], sy[NJ];
#pragma unroll
  for (int jb = 0; jb < NJ; ++jb) {
    if (a.job[jb].src_layout == kTokenMajor) {
      sx[jb] = h * D;
      sy[jb] = b * d.Lq + f * d.T_f + row0;
    } else {
      sx[jb] = 0;
      sy[jb] = (bh * d.Fc + f) * d.T_pad + row0;
    }
  }
  auto issue = [&](int q) {  // group q into buffer q & 1
    uint8_t* buf = rp_smem + (q & 1) * kBuf;
    mbar_arrive_expect_tx(&bar[q & 1], kBuf);
#pragma unroll
    for (int jb = 0; jb < NJ; ++jb) tma_load_2d(buf + jb * L::kTile, maps[jb], &bar[q & 1], sx[jb], sy[jb] + q * L::kRows);
    if (kTab) tma_load_2d(buf + NJ * L::kTile, &mt, &bar[q & 1], L::kTabX, row0 + q * L::kRows);
  };
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    *abort_flag = 0;
    fence_barrier_init();
    issue(0);
    if (ngroups > 1) issue(1);
  }

  JobRows jr[NJ];
#pragma unroll
  for (int jb = 0; jb < NJ; ++jb) jr[jb] = job_rows<D>(a.job[jb], d, b, h, bh, f, slot, a.W, row0 + rg, cgi * 8);
  int axis[4];
  float ct[4], st[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int p = cgi * 4 + i;
    axis[i] = p < a.tab.pt ? 0 : 1;
    ct[i] = 1.f;
    st[i] = 0.f;
    if (kAnyRot && p < a.tab.pt) {
      ct[i] = __ldg(a.tab.cos_t + (size_t)t * a.tab.pt + p);
      st[i] = __ldg(a.tab.sin_t + (size_t)t * a.tab.pt + p);
    }
  }
  const bool spatial = cgi * 8 >= L::kTabX;  // this thread's pairs are in the table tile
  float acc[2][8];
#pragma unroll
  for (int jb = 0; jb < 2; ++jb)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[jb][i] = 0.f;
  __syncthreads();  // barriers initialised

  for (int q = 0; q < ngroups; ++q) {
    const uint8_t* buf = rp_smem + (q & 1) * kBuf;
    const uint16_t* tile = reinterpret_cast<const uint16_t*>(buf);
    const float* ttab = reinterpret_cast<const float*>(buf + NJ * L::kTile);
    mbar_wait(&bar[q & 1], (q >> 1) & 1, abort_flag, a.err);
    __syncthreads();
    if (*abort_flag) break;  // read after the barrier: the same for every thread
    const int g = q * L::kRows;
#pragma unroll
    for (int p = 0; p < kPass; ++p) {
      const int rl = p * kRP + rg;  // row in the group
      const bool live = g + rl < valid;
      float c[4], s[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        c[i] = ct[i];
        s[i] = st[i];
      }
      if (kTab && spatial) {
        const float4* e = reinterpret_cast<const float4*>(ttab + rl * L::kTabW + 8 * cgi - L::kTabX);
        const float4 e0 = e[0], e1 = e[1];
        const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (axis[i] != 0) {
            c[i] = ev[2 * i];
            s[i] = ev[2 * i + 1];
          }
        }
      }
#pragma unroll
      for (int jb = 0; jb < NJ; ++jb) {
        uint4 y = make_uint4(0u, 0u, 0u, 0u);
        if (live) {
          y = *reinterpret_cast<const uint4*>(tile + (jb * L::kRows + rl) * D + cgi * 8);
          if (kRot[jb]) y = rotate4(y, c, s);
        }
        if (kPool[jb]) pool_add(acc[jb], y);
        if (jr[jb].dst && (live || !jr[jb].tok_dst))
          *reinterpret_cast<uint4*>(jr[jb].dst + (size_t)(g + p * kRP) * jr[jb].dstride) = y;
      }
    }
    if (q + 2 < ngroups) {  // buffer q & 1 was read: hand it back to the async proxy for group q + 2
      fence_proxy_async_smem();
      __syncthreads();
      if (tid == 0) issue(q + 2);
    }
  }

  // block means, reduced over the rows in a fixed order (exchange in buffer 0)
  __syncthreads();
#pragma unroll
  for (int jb = 0; jb < 2; ++jb) {
    if (!kPool[jb] || jb >= NJ) continue;
    warp_col_sums<D>(acc[jb], red, tid);
    __syncthreads();
    if (tid < D && !*abort_flag) {
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) sum += red[w * D + tid];
      const StreamJob& job = a.job[jb];
      size_t off;
      if (job.pool_layout == kPoolChunk) {
        off = ((size_t)bh * d.NQB + (size_t)f * d.nb + j) * D + tid;
      } else {
        off = (((size_t)bh * a.W + slot) * d.nb + j) * D + tid;
      }
      job.pool[off] = sum / (float)valid;
    }
    __syncthreads();
  }
}

// Frame means from block means: sum_j count_j * mean_j / T_f, in block order
// (for block means written by the fused QKV projection).
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

// TMA descriptors of the staged kernel; false if a tensor cannot be described.
template <int D, int NJ>
static bool rope_maps(const RopePoolArgs& a, bool tok, CUtensorMap (&m)[4]) {
  using L = RopeTma<D>;
  const Dims& d = a.d;
  for (int jb = 0; jb < 3; ++jb) {
    const StreamJob& job = a.job[jb < NJ ? jb : 0];
    bool ok;
    if (job.src_layout == kTokenMajor) {
      ok = make_map_2d(&m[jb], job.src, false, (uint64_t)d.H * D, (uint64_t)d.B * d.Lq, (uint64_t)d.H * D * 2, D,
                       L::kRows);
    } else {
      ok = make_map_2d(&m[jb], job.src, false, D, (uint64_t)d.B * d.H * d.Fc * d.T_pad, (uint64_t)D * 2, D,
                       L::kRows);
    }
    if (!ok) return false;
  }
  m[3] = m[0];
  if (tok)
    return make_map_2d(&m[3], a.tab.cs_tok, true, D, (uint64_t)d.Fh * a.tab.tab_w, (uint64_t)D * 4, L::kTabW,
                       L::kRows);
  return true;
}

template <int D, int NJ, int FL>
static cudaError_t launch_rope_pool_t(const RopePoolArgs& a, cudaStream_t stream) {
  using L = RopeTma<D>;
  constexpr bool kAnyRot = (FL & (kRot0 | kRot1)) != 0;
  dim3 grid(a.d.Fc * a.d.nb, a.d.B * a.d.H);
  // the staged kernel reads the per-position table as rows of the frame (w fastest)
  const bool tok = kAnyRot && a.tab.cs_tok != nullptr && a.tab.tab_w == a.d.Fw;
  CUtensorMap m[4];
  if ((!kAnyRot || tok) && rope_maps<D, NJ>(a, tok, m)) {
    const int smem = 2 * L::buf_bytes(NJ, tok) + 32;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static bool attr[2][64] = {};  // per device: the shared-memory limit was raised
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (tok) {
      if (!attr[1][dev]) {
        e = cudaFuncSetAttribute(rope_pool_tma_kernel<D, NJ, FL, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem);
        if (e != cudaSuccess) return e;
        attr[1][dev] = true;
      }
      rope_pool_tma_kernel<D, NJ, FL, true><<<grid, 256, smem, stream>>>(m[0], m[1], m[2], m[3], a);
    } else if constexpr (!kAnyRot) {
      if (!attr[0][dev]) {
        e = cudaFuncSetAttribute(rope_pool_tma_kernel<D, NJ, FL, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem);
        if (e != cudaSuccess) return e;
        attr[0][dev] = true;
      }
      rope_pool_tma_kernel<D, NJ, FL, false><<<grid, 256, smem, stream>>>(m[0], m[1], m[2], m[3], a);
    }
    return cudaGetLastError();
  }
  // tables without the per-position expansion: per-row lookups, loads into registers
  constexpr int kRows = D == 128 ? 16 : 32;  // one pass of 256 threads
  rope_pool_kernel<D, NJ, FL, kRows, 3><<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_rope_pool_d(const RopePoolArgs& a, int fl, cudaStream_t stream) {
  switch (a.njobs * 16 + fl) {
    // chunk call: Q rotated (pooled when sparse), K rotated and pooled, V copied
    case 3 * 16 + (kRot0 | kRot1 | kPool1): return launch_rope_pool_t<D, 3, kRot0 | kRot1 | kPool1>(a, stream);
    case 3 * 16 + (kRot0 | kRot1 | kPool0 | kPool1):
      return launch_rope_pool_t<D, 3, kRot0 | kRot1 | kPool0 | kPool1>(a, stream);
    // append: K (rotated or not) pooled, V copied
    case 2 * 16 + (kRot0 | kPool0): return launch_rope_pool_t<D, 2, kRot0 | kPool0>(a, stream);
    case 2 * 16 + kPool0: return launch_rope_pool_t<D, 2, kPool0>(a, stream);
    // rotation alone; pooling alone
    case 1 * 16 + kRot0: return launch_rope_pool_t<D, 1, kRot0>(a, stream);
    case 1 * 16 + kPool0: return launch_rope_pool_t<D, 1, kPool0>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_rope_pool(const RopePoolArgs& a, cudaStream_t stream) {
  if (a.njobs < 1 || a.njobs > 3) return cudaErrorInvalidValue;
  if ((int64_t)a.d.B * a.d.H > 65535) return cudaErrorInvalidConfiguration;
  if (a.njobs == 3 && (a.job[2].pool || a.job[2].rotate)) return cudaErrorInvalidValue;
  int fl = 0;
  for (int jb = 0; jb < a.njobs && jb < 2; ++jb) {
    if (a.job[jb].rotate) fl |= jb == 0 ? kRot0 : kRot1;
    if (a.job[jb].pool) fl |= jb == 0 ? kPool0 : kPool1;
  }
  return a.d.D == 128 ? launch_rope_pool_d<128>(a, fl, stream) : launch_rope_pool_d<64>(a, fl, stream);
}

cudaError_t launch_frame_pool(const FramePoolArgs& a, cudaStream_t stream) {
  dim3 grid(a.d.Fc, a.d.B * a.d.H);
  frame_pool_kernel<<<grid, a.d.D, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace cva
