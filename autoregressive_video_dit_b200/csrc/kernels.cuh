// Kernel argument blocks and launchers of libcva (host <-> kernel files).
#pragma once

#include "cva_internal.cuh"

namespace cva {

// Launches `kernel`; with `dependent`, as a programmatic dependent launch
// (the kernel must call griddep_wait() before it touches memory that the
// previous work on the stream reads or writes).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t stream, bool dependent, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---- steps 1-3: rotary embedding, cache append, pooling (rope_pool.cu) ----
enum : int { kTokenMajor = 0, kHeadMajor = 1, kCacheSlots = 2 };
enum : int { kPoolNone = 0, kPoolChunk = 1, kPoolCache = 2 };

struct StreamJob {
  const uint16_t* src;  // bf16 input
  int src_layout;       // kTokenMajor or kHeadMajor
  uint16_t* dst;        // bf16 output (nullptr: none)
  int dst_layout;       // kTokenMajor, kHeadMajor or kCacheSlots
  int rotate;           // apply the rotary embedding
  float* pool;          // block means (nullptr: none)
  int pool_layout;      // kPoolChunk or kPoolCache
};

struct RopePoolArgs {
  StreamJob job[3];
  int njobs;
  int* err;      // device error word (bounded waits of the staged kernel)
  RopeTab tab;
  Dims d;
  int t0;
  int W;
};

struct FramePoolArgs {
  const float* blk_pool;
  float* frm_pool;
  int layout;  // kPoolChunk: [bh][NQB][D] -> [bh][Fc][D]; kPoolCache: [bh][W][nb][D] -> [bh][W][D]
  Dims d;
  int t0;
  int W;
};

cudaError_t launch_rope_pool(const RopePoolArgs& a, cudaStream_t stream);
cudaError_t launch_frame_pool(const FramePoolArgs& a, cudaStream_t stream);

// ---- step 4: selection (hsa_select.cu) ----------------------------------
struct SelectArgs {
  const float* qpool;      // [B][H][NQB][D]
  const float* kpool_blk;  // [B][H][W][nb][D]
  const float* kpool_frm;  // [B][H][W][D]
  int32_t* frame_idx;      // [B][H][NQB][k_f_stride] or nullptr
  int32_t* block_idx;      // [B][H][NQB][k_b_max]
  int32_t* block_cnt;      // [B][H][NQB]
  Dims d;
  int W, t_lo, F;          // history frames t_lo .. t_lo+F-1
  int k_f, k_b, k_f_stride, k_b_max;
  // Top-p budget of the second level (0: top-k with k = k_b). With p > 0,
  // k_b is the cap and the blocks are taken in rank order while the softmax
  // mass (temperature sqrt(D), weighted by token counts) ranked above them
  // is below p times the total.
  float topp;
  float temp_log2;         // log2(e) / sqrt(D)
};
cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream, bool dependent = false);
// Pairs each head's 64-row query blocks into 128-row attention tiles by the
// overlap of their picked frames (hsa_select.cu).
cudaError_t launch_pair_query_blocks(const int32_t* frame_idx, int kfe, const Dims& d, int t_lo, int F,
                                     int MT, int32_t* qpair, cudaStream_t stream, bool dependent = false);

// ---- step 5: attention (attn_sm100.cu) -----------------------------------
struct AttnArgs {
  const int32_t* block_idx;  // [B][H][NQB][k_b_max] or nullptr (dense)
  const int32_t* block_cnt;  // [B][H][NQB]
  int k_b_max;
  uint16_t* out;             // bf16 [B, Lq, H, D]
  float* lse;                // [B][H][Lq] or nullptr
  int* err;                  // device error word
  Dims d;
  int W, t0, t_lo, F;
  int MT;                    // 128-row query tiles per (b, h)
  float scale_log2;          // log2(e) / sqrt(D)
  // Tail split: tiles 0 .. Qf-1 (b*h major, tile minor) run whole; each
  // later tile is cut into `pieces` key ranges whose partial (O, max, sum)
  // go to part_o / part_ml and are combined by a merge launch.
  int Qf, pieces;
  float* part_o;             // [piece slot][128][D] fp32, unnormalised
  float* part_ml;            // [piece slot][128][2] running max (log2 units), sum
  // Query blocks held by each 128-row tile when blocks are 64 rows:
  // [B*H][MT][2] (rows 0-63, rows 64-127; -1 for none), or nullptr for the
  // blocks 2m and 2m+1 of tile m.
  const int32_t* qpair;
  // Optional: frame means of the chunk's cache frames (t0 .. t0+Fc-1) from
  // their block means, computed by the CTAs' spare warps.
  const float* kpool_blk;    // [B][H][W][nb][D]
  float* kpool_frm;          // [B][H][W][D], or nullptr
};
// Piece slots of the tail split (one per SM at most).
constexpr int kAttnMaxPieces = 160;
constexpr int kAttnMaxEntries = 4096;     // 64-row key units per CTA (two query tiles)
constexpr int kAttnMaxBitmapWords = 256;  // history blocks per CTA <= 8192

// Builds the tensor maps and launches the attention kernel.
cudaError_t launch_attention(const AttnArgs& a, const void* q_rot, const void* cache_k,
                             const void* cache_v, cudaStream_t stream, const char** why,
                             bool dependent = false);

// Tiled TMA descriptor of a bf16 tensor [d2][d1][d0] (d0 innermost) with a
// box of 64 x box1 elements and 128-byte swizzle (attn_sm100.cu).
bool make_map(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box1);
// Tiled TMA descriptor of a 2D bf16 (or fp32) tensor [d1][d0] with rows of
// row_bytes, a box of box0 x box1 elements and no swizzle (attn_sm100.cu).
bool make_map_2d(CUtensorMap* map, const void* base, bool fp32, uint64_t d0, uint64_t d1,
                 uint64_t row_bytes, uint32_t box0, uint32_t box1);

// ---- head-sharded path: batched row copies (shard.cu) -------------------
struct RowCopy2D {
  int64_t n0, n1, inner;    // rows i0 < n0, i1 < n1 of `inner` bytes
  int64_t ss0, ss1;         // source strides (bytes)
  int64_t ds0, ds1;         // destination strides (bytes)
};
cudaError_t launch_copy_rows_2d(const void* src, void* dst, const RowCopy2D& c, cudaStream_t stream);

// ---- QKV projection + Causal-RoPE + append + block pooling (qkv_rope.cu) --
struct QkvArgs {
  Dims d;
  int C;                     // hidden size (multiple of 64)
  int t0, W;                 // chunk start frame, cache window
  RopeTab tab;
  uint16_t* q_rot;           // [B][H][Fc*T_pad][D]
  uint16_t* k_cache;         // [B][H][W][T_pad][D]
  uint16_t* v_cache;
  float* qpool;              // [B][H][NQB][D] block means of q_rot, or nullptr
  float* kpool_blk;          // [B][H][W][nb][D] block means of k_rot
  int MT;                    // 128-row tiles over the padded rows of the chunk
  int NT;                    // 256-column tiles over the 3*H*D projection outputs
  int* err;
};
cudaError_t launch_qkv_rope(const QkvArgs& a, const void* x, const void* w, cudaStream_t stream,
                            const char** why);

// Sets the thread-local message cva_last_error() returns; returns `code`.
int report_error(int code, const char* msg);

// Host checks of cva_chunk_attention's arguments other than the workspace
// (same codes and messages); *ws_need gets the workspace bytes it needs.
int check_chunk_call(const void* q, const void* k, const void* v, const cva_kv_cache* cache,
                     const cva_rope_tables* tables, int32_t t0, int32_t k_f, int32_t k_b,
                     const void* out, size_t* ws_need);

// ---- diagnostics (diag.cu) ------------------------------------------------
cudaError_t launch_wait_timeout(int* err, int* result, uint64_t limit_ns, cudaStream_t stream);
cudaError_t launch_mma_cycles(int M, int N, int iters, unsigned long long* cycles, int sms, int* err,
                              cudaStream_t stream);

}  // namespace cva
