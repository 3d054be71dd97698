/*
 * cva.h -- C ABI of the per-chunk attention path of a causal, chunk-by-chunk
 * autoregressive video diffusion transformer, for NVIDIA B200 (sm_100a).
 *
 * For every new chunk of Fc latent frames the path
 *   1. rotates Q and K with a 3D rotary embedding whose temporal coordinate
 *      is a global time index (cva_rope3d_precompute, cva_rope3d_apply);
 *   2. appends the rotated K and V to a chunk-causal, optionally rolling,
 *      frame cache (cva_kv_append);
 *   3. mean-pools Q and K per block and per frame (cva_hsa_compress; the K
 *      pools are produced by cva_kv_append and kept with the cache);
 *   4. picks, per query block, the top frames by frame-pooled keys and then
 *      the top blocks inside them by block-pooled keys (cva_hsa_select);
 *   5. runs block-sparse flash attention over the picked history blocks plus
 *      the whole current chunk (cva_blocksparse_attn_fwd).
 * cva_chunk_attention runs 1-5 back to back; cva_cag_budget turns a chunk
 * index into the (k_f, k_b) budget.
 *
 * Conventions
 *   - Notation: B batch, H heads, D head_dim, Fh x Fw latent grid,
 *     T_f = Fh*Fw tokens per frame, blk block size, nb = ceil(T_f/blk)
 *     blocks per frame, T_pad = nb*blk, Fc frames per chunk, Lq = Fc*T_f
 *     queries per chunk, NQB = Fc*nb query blocks, W frame slots.
 *   - Blocks are per frame: block j of a frame holds tokens
 *     [j*blk, min((j+1)*blk, T_f)); the last block of a frame may be short.
 *   - Tokens of a chunk are ordered frame-major, then row-major (h, w).
 *   - Tensors marked bf16 are IEEE bfloat16 (uint16 storage). Every pointer
 *     is a DEVICE pointer unless marked HOST. The caller allocates all
 *     memory (the library never allocates, frees or synchronises) and owns
 *     it; the library keeps no pointer after a call returns.
 *   - Every call validates its arguments on the host before launching
 *     anything and returns CVA_OK (0) or a negative CVA_E* code; the
 *     thread-local message of the last failure is cva_last_error().
 *     Kernels run asynchronously on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream); errors found on the device (a bad index, a
 *     wait that timed out) are latched in a device word that
 *     cva_device_status() reads.
 *   - Supported: D in {64, 128}, blk in {64, 128}, B*H <= 65535,
 *     k_f * nb <= 1024, history frames <= 256.
 *
 * Sources. "Accelerating Video Generation Inference with Sequential-Parallel
 * 3D Positional Encoding Using a Global Time Index" (section 2B: global
 * time index t + s; section 2C: precomputed cos/sin tables, fused RoPE) and
 * "Light Forcing" (section 2.1: Chunk-Aware Growth budget; section 2.2:
 * Hierarchical Sparse Attention -- block/frame mean pooling, frame then
 * block selection, attention over the picked frame-block pairs).
 */
#ifndef CVA_H_
#define CVA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CVA_VERSION 1

/* Status codes. */
enum {
  CVA_OK = 0,
  CVA_EINVAL = -1,   /* null pointer, bad shape or argument */
  CVA_ENOTSUP = -2,  /* head_dim or block size the kernels do not support */
  CVA_ERANGE = -3,   /* t0 beyond the tables, budget beyond the candidates */
  CVA_ENOMEM = -4,   /* a caller buffer (workspace, cache arena) is too small */
  CVA_ELAUNCH = -5,  /* a CUDA call failed; cva_last_error() has its string */
  CVA_EDEVICE = -6   /* the device latched an error (see cva_device_status) */
};

/* Device-side error codes latched by the kernels (first error wins). */
enum {
  CVA_DEV_OK = 0,
  CVA_DEV_TIMEOUT = 1,     /* a pipeline wait exceeded its time limit */
  CVA_DEV_BAD_INDEX = 2,   /* a block index outside the cache window */
  CVA_DEV_BAD_COUNT = 3    /* a block count above k_b_max */
};

typedef void* cva_stream_t; /* cudaStream_t */

/* Problem shape (host struct). */
typedef struct cva_shape {
  int32_t batch;        /* B  >= 1 */
  int32_t heads;        /* H  >= 1 */
  int32_t head_dim;     /* D  in {64, 128} */
  int32_t frame_h;      /* Fh >= 1 */
  int32_t frame_w;      /* Fw >= 1 */
  int32_t chunk_frames; /* Fc >= 1 */
  int32_t block;        /* blk in {64, 128} */
} cva_shape;

/* Rotary table configuration (host struct). */
typedef struct cva_rope_cfg {
  int32_t head_dim;     /* D */
  int32_t max_t;        /* rows of the temporal table: global t < max_t */
  int32_t frame_h;      /* rows of the height table */
  int32_t frame_w;      /* rows of the width table */
  double theta;         /* base, 10000 for the video DiT */
} cva_rope_cfg;

/* Device copies of the rotary tables (host struct holding device pointers).
 * Each table is fp32 row-major [positions][pairs of that axis]. cs_tok is
 * optional (NULL: not used): the spatial tables expanded per position,
 * (cos, sin) interleaved, [frame_h][frame_w][head_dim/2][2] floats with
 * (1, 0) for the temporal pairs (cva_rope3d_precompute_tokens), 16-byte
 * aligned; with it the rotation reads one contiguous 32-byte entry per 4
 * pairs instead of looking each pair up. Results are identical. */
typedef struct cva_rope_tables {
  const float* cos_t; const float* sin_t;   /* [max_t][p_t]   */
  const float* cos_h; const float* sin_h;   /* [frame_h][p_h] */
  const float* cos_w; const float* sin_w;   /* [frame_w][p_w] */
  int32_t max_t, frame_h, frame_w, head_dim;
  const float* cs_tok;                      /* [frame_h][frame_w][head_dim/2][2] or NULL */
} cva_rope_tables;

/* Frame cache of one attention layer (host struct holding device pointers).
 * Frame with global index t lives in slot (t mod window). Rows j*blk+r with
 * r >= valid rows of the frame's last block are zero. Filled by
 * cva_kv_cache_init; the caller owns the arena. */
typedef struct cva_kv_cache {
  void* k;            /* bf16 [B][H][window][T_pad][D], rotated keys     */
  void* v;            /* bf16 [B][H][window][T_pad][D], values           */
  float* kpool_blk;   /* fp32 [B][H][window][nb][D], block-mean keys     */
  float* kpool_frm;   /* fp32 [B][H][window][D], frame-mean keys         */
  int32_t window;     /* W frame slots (>= Fc)                          */
  int32_t t_begin;    /* global index of the stream's first frame       */
  cva_shape shape;
} cva_kv_cache;

/* Chunk-Aware Growth schedule ("Light Forcing", section 2.1), exact
 * rationals: density d_i = d_base + d_slope * (i - pivot), clamped to
 * [0, 1]; k_f = min(k_f_max, history frames); k_b = min(k_f * nb,
 * floor(d_i * history_blocks + 1/2)), or min(k_f * nb, k_b_fixed) when
 * k_b_fixed >= 0. dense != 0, chunk 1 or an empty history keep everything. */
typedef struct cva_cag_cfg {
  int32_t dense;
  int32_t k_f_max;
  int64_t d_base_num, d_base_den;
  int64_t d_slope_num, d_slope_den;
  int32_t pivot;
  int32_t k_b_fixed;  /* -1: use the density */
} cva_cag_cfg;

/* ---- library ------------------------------------------------------------ */

int cva_version(void);
/* Message of the last failed call on this host thread ("" if none). */
const char* cva_last_error(void);
/* Reads (and with clear != 0 resets) the device error word of the current
 * device into *code. Synchronises the device. */
int cva_device_status(int32_t* code, int32_t clear);

/* ---- 0. rotary tables (Causal-RoPE SP, section 2C) ----------------------- */

/* Pairs per axis: p_h = p_w = (D/2)/3, p_t = D/2 - 2*p_h (D=128: 22/21/21). */
int cva_rope_axis_pairs(int32_t head_dim, int32_t* p_t, int32_t* p_h, int32_t* p_w);

/* Fills HOST buffers with cos/sin(pos * theta^(-j/p_a)) for every position
 * pos < rows of the axis and pair j < p_a, computed in double and stored as
 * float: cos_t/sin_t [max_t][p_t], cos_h/sin_h [frame_h][p_h], cos_w/sin_w
 * [frame_w][p_w]. The caller copies them to the device once. */
int cva_rope3d_precompute(const cva_rope_cfg* cfg, float* cos_t, float* sin_t,
                          float* cos_h, float* sin_h, float* cos_w, float* sin_w);

/* Fills the HOST buffer cs_tok [frame_h][frame_w][head_dim/2][2] with the
 * (cos, sin) of every spatial pair at every (h, w) position, the same floats
 * as the per-axis tables, and (1, 0) for the temporal pairs. */
int cva_rope3d_precompute_tokens(const cva_rope_cfg* cfg, float* cs_tok);

/* ---- 1. rotary embedding with a global time index (section 2B) ----------- */

/* y = RoPE(x) for one chunk starting at global frame t0: token n of the
 * chunk has t = t0 + n / T_f, h = (n mod T_f) / Fw, w = n mod Fw; pair
 * (x[2p], x[2p+1]) is rotated by the angle of its axis (pairs [0, p_t) use
 * t, the next p_h use h, the last p_w use w). fp32 arithmetic, bf16 I/O.
 *   x: bf16 [B, Lq, H, D].
 *   out_layout 0: y bf16 [B, Lq, H, D];
 *   out_layout 1: y bf16 [B][H][Fc*T_pad][D] (frame f, token r at row
 *                 f*T_pad + r), pad rows written as zero.
 * CVA_ERANGE if t0 + Fc > tables->max_t or t0 < 0. */
int cva_rope3d_apply(const void* x, void* y, const cva_rope_tables* tables,
                     const cva_shape* shape, int32_t t0, int32_t out_layout,
                     cva_stream_t stream);

/* ---- 2. cache append (+ K pooling of step 3) ----------------------------- */

/* "Accelerating Video Generation Inference with Sequential-Parallel 3D
 * Positional Encoding Using a Global Time Index", section 1 (problem): the
 * Self-Forcing style generator produces the video chunk by chunk, caching the
 * keys and values of earlier chunks (KV caching) in a rolling window; the
 * keys are cached already rotated with their global time index (section 2B).
 * Writes the chunk's frames t0 .. t0+Fc-1 into their slots: K rotated (or
 * copied as is when tables == NULL, for keys rotated upstream), V copied,
 * pad rows zeroed, and the block-mean and frame-mean of the stored (bf16)
 * keys written to kpool_blk / kpool_frm in fp32.
 *   k, v: bf16 [B, Lq, H, D].
 * The slots overwritten are those of frames t0+f-W (rolling eviction). */
int cva_kv_append(const void* k, const void* v, const cva_kv_cache* cache,
                  const cva_rope_tables* tables, int32_t t0, cva_stream_t stream);

/* History frames a chunk at t0 sees: [max(t_begin, t0 + Fc - W), t0) -- the
 * cached earlier frames still inside the rolling window of W frames (the same
 * section 1 passage as cva_kv_append: KV caching with a rolling window). */
int cva_history_frames(const cva_kv_cache* cache, int32_t t0, int32_t* t_lo,
                       int32_t* count);

/* ---- 3. query pooling ("Light Forcing" 2.2, token compression) ---------- */

/* Block means (over each block's valid tokens) and frame means (over the
 * frame's T_f tokens) of rotated queries, fp32 accumulation in a fixed order.
 *   q_rot: bf16 [B][H][Fc*T_pad][D] (out_layout 1 of cva_rope3d_apply).
 *   qpool_blk: fp32 [B][H][NQB][D], query block qb = f*nb + j.
 *   qpool_frm: fp32 [B][H][Fc][D], or NULL. */
int cva_hsa_compress(const void* q_rot, const cva_shape* shape, float* qpool_blk,
                     float* qpool_frm, cva_stream_t stream);

/* ---- 4. two-level selection ("Light Forcing" 2.2) ------------------------ */

/* For every (b, h, query block): scores q.kf of the history frames with the
 * block-pooled query q; the top k_f (all when history <= k_f) by score, ties
 * to the lower t; then scores q.kb of every block of those frames, the top
 * k_b over all of them, ties to the lower (t, j).
 *   frame_idx: int32 [B][H][NQB][k_f_eff] global t, ascending
 *              (k_f_eff = min(k_f, history frames)); may be NULL.
 *   block_idx: int32 [B][H][NQB][k_b] ids t*nb + j, ascending.
 *   block_cnt: int32 [B][H][NQB] number of valid entries (= k_b).
 * CVA_ERANGE if k_b > k_f_eff * nb, k_f < 1 with a history, or k_b < 0. */
int cva_hsa_select(const float* qpool_blk, const cva_kv_cache* cache, int32_t t0,
                   int32_t k_f, int32_t k_b, int32_t* frame_idx, int32_t* block_idx,
                   int32_t* block_cnt, cva_stream_t stream);

/* Top-p budget for the second level ("Sparse VideoGen2", section B: clusters
 * sorted by estimated attention and taken until the cumulative share reaches
 * p). Frames as cva_hsa_select; the candidate blocks of the picked frames
 * are ranked by q.kb (ties to the lower (t, j)); block c's estimated share is
 * its valid token count n_c (blk, or the frame's tail for its last block)
 * times exp((s_c - s_max) / sqrt(D)), over the sum of them all (fp32,
 * exp2f). In rank order a block is taken while the share ranked above it is
 * below p: the top block always, at most k_cap blocks.
 *   block_idx: int32 [B][H][NQB][k_cap], the first block_cnt entries valid
 *              (ascending ids t*nb + j); the rest are not written.
 *   block_cnt: int32 [B][H][NQB], 1 .. k_cap (0 without history).
 * CVA_ERANGE if p is outside (0, 1], k_cap < 1 or k_cap > k_f_eff * nb.
 * cva_blocksparse_attn_fwd takes these lists with k_b_max = k_cap. */
int cva_hsa_select_topp(const float* qpool_blk, const cva_kv_cache* cache, int32_t t0,
                        int32_t k_f, int32_t k_cap, float p, int32_t* frame_idx,
                        int32_t* block_idx, int32_t* block_cnt, cva_stream_t stream);

/* ---- 5. block-sparse flash attention ("Light Forcing" 2.2, execution) ---- */

/* For query i of query block qb: key set S = valid tokens of the history
 * blocks block_idx[b][h][qb][0 .. block_cnt-1] plus every token of the
 * current chunk (frames t0 .. t0+Fc-1, already appended);
 *   o_i = sum_{j in S} softmax_j(q_i . k_j / sqrt(D)) v_j,
 *   lse_i = log sum_{j in S} exp(q_i . k_j / sqrt(D)).
 * block_idx == NULL: every history frame's every block (dense).
 *   q_rot: bf16 [B][H][Fc*T_pad][D]; out: bf16 [B, Lq, H, D];
 *   lse: fp32 [B][H][Lq] or NULL.
 *   workspace: device scratch of cva_attn_workspace_bytes() bytes (256-byte
 *   aligned), or NULL. With it, the query tiles of the last, partial wave of
 *   CTAs are cut into key-range pieces that fill the SMs and are merged by a
 *   second launch (same result up to fp32 rounding order); without it every
 *   tile runs whole. A smaller ws_bytes counts as NULL.
 * Tensor cores (tcgen05, accumulators in tensor memory), TMA tile loads
 * gathered by block index, fp32 online softmax. */
int cva_attn_workspace_bytes(const cva_shape* shape, int32_t k_b_max, size_t* bytes);
int cva_blocksparse_attn_fwd(const void* q_rot, const cva_kv_cache* cache, int32_t t0,
                             const int32_t* block_idx, const int32_t* block_cnt,
                             int32_t k_b_max, void* out, float* lse, void* workspace,
                             size_t ws_bytes, cva_stream_t stream);

/* ---- QKV projection fused with steps 1-3 ----------------------------------
 * "Accelerating Video Generation Inference with Sequential-Parallel 3D
 * Positional Encoding Using a Global Time Index", section 2C (operator
 * fusion: the QKV projection and Causal-RoPE in one kernel) with the global
 * time index of section 2B.
 *
 * y = x W^T for the chunk's tokens, on the tensor cores (fp32 accumulate):
 *   x:     bf16 [B, Lq, C], C = hidden (a multiple of 64, >= 64);
 *   w_qkv: bf16 [3*H*D, C], rows: q heads 0..H-1 (D rows each), then the k
 *          heads, then the v heads; no bias.
 * q and k are rotated like cva_rope3d_apply (temporal coordinate t0 + f),
 * in fp32 from the accumulator, and rounded once to bf16. Writes
 *   q_rot:     bf16 [B][H][Fc*T_pad][D], pad rows zero (the attention's Q);
 *   qpool_blk: fp32 [B][H][NQB][D] block means of the stored q, or NULL;
 * and appends k and v to the cache slots of frames t0 .. t0+Fc-1 exactly as
 * cva_kv_append does (pad rows zero, block and frame means of the stored
 * k). x, w_qkv and q_rot must be 16-byte aligned. Two launches: the fused
 * projection kernel and the frame pooling of the new cache frames. */
int cva_qkv_rope_append(const void* x, const void* w_qkv, int32_t hidden,
                        const cva_kv_cache* cache, const cva_rope_tables* tables,
                        int32_t t0, void* q_rot, float* qpool_blk, cva_stream_t stream);

/* ---- fused chunk call ---------------------------------------------------- */

/* Steps 1-5 for one chunk, in the order "Light Forcing" section 2.2 gives
 * them (token compression by mean pooling, frame then block selection, then
 * attention over the picked frame-block pairs) after the rotation with the
 * global time index of "Accelerating Video Generation Inference with
 * Sequential-Parallel 3D Positional Encoding Using a Global Time Index",
 * section 2B: RoPE(Q) with Q pooling, RoPE(K)+append+K pooling,
 * selection with (k_f, k_b) (dense when k_f < 0), attention. The launches,
 * in stream order: the rotate/append/pool kernel (Q, K and V in one pass),
 * the selection (sparse only), the attention (whose spare warps also write
 * the frame means of the new cache frames), the merge of split tail tiles
 * (only when the query tiles leave a partial wave). Results equal the staged
 * calls' up to fp32 rounding order.
 *   q, k, v: bf16 [B, Lq, H, D]; out: bf16 [B, Lq, H, D]; lse: fp32
 *   [B][H][Lq] or NULL. workspace: cva_chunk_workspace_bytes() bytes. */
int cva_chunk_workspace_bytes(const cva_shape* shape, int32_t k_f, int32_t k_b,
                              size_t* bytes);
int cva_chunk_attention(const void* q, const void* k, const void* v,
                        const cva_kv_cache* cache, const cva_rope_tables* tables,
                        int32_t t0, int32_t k_f, int32_t k_b, void* workspace,
                        size_t ws_bytes, void* out, float* lse, cva_stream_t stream);

/* cva_chunk_attention (same passages: "Light Forcing" section 2.2 and the
 * global time index of section 2B of the Causal-RoPE page) with the top-p
 * block budget of cva_hsa_select_topp ("Sparse VideoGen2", section B)
 * (k_f >= 1, cap k_cap, threshold p in (0, 1]); workspace:
 * cva_chunk_workspace_bytes(shape, k_f, k_cap) bytes. */
int cva_chunk_attention_topp(const void* q, const void* k, const void* v,
                             const cva_kv_cache* cache, const cva_rope_tables* tables,
                             int32_t t0, int32_t k_f, int32_t k_cap, float p, void* workspace,
                             size_t ws_bytes, void* out, float* lse, cva_stream_t stream);

/* Steps 1-3 of cva_chunk_attention alone, in its single launch ("Light
 * Forcing" section 2.2 token compression and the global time index of
 * section 2B of the Causal-RoPE page): Q rotated with global time t0 into
 * q_rot and, when qpool_blk is not NULL, its block means; K rotated and V
 * copied into the cache slots of frames t0 .. t0+Fc-1 (rolling eviction as
 * cva_kv_append), with the block means of the stored keys. The frame means
 * of the new frames are not written: cva_chunk_attention writes them in its
 * attention launch, and cva_kv_frame_means writes them for callers that
 * run their own attention.
 *   q, k, v: bf16 [B, Lq, H, D] (16-byte aligned);
 *   q_rot: bf16 [B][H][Fc*T_pad][D] (out_layout 1 of cva_rope3d_apply);
 *   qpool_blk: fp32 [B][H][NQB][D] or NULL.
 * tables must hold the per-position table (cva_rope3d_precompute_tokens).
 * Errors as cva_chunk_attention's. */
int cva_rotate_append_pool(const void* q, const void* k, const void* v,
                           const cva_kv_cache* cache, const cva_rope_tables* tables,
                           int32_t t0, void* q_rot, float* qpool_blk, cva_stream_t stream);

/* Frame means (fp32, over each frame's T_f tokens, fixed order) of the
 * cached keys of frames t0 .. t0+Fc-1 from their block means ("Light
 * Forcing" section 2.2: frame-pooled keys); completes cva_rotate_append_pool
 * for callers that do not follow it with cva_chunk_attention. */
int cva_kv_frame_means(const cva_kv_cache* cache, int32_t t0, cva_stream_t stream);

/* Steps 1-5 for one chunk starting from the hidden states: the fused QKV
 * projection with Causal-RoPE, append and pooling (cva_qkv_rope_append, the
 * pages' section 2C operator fusion), then selection with (k_f, k_b)
 * (dense when k_f < 0) and attention, all on the caller's stream.
 *   x: bf16 [B, Lq, C]; w_qkv: bf16 [3*H*D, C] (as cva_qkv_rope_append);
 *   out: bf16 [B, Lq, H, D]; lse: fp32 [B][H][Lq] or NULL;
 *   workspace: cva_chunk_workspace_bytes() bytes (256-byte aligned). */
int cva_chunk_attention_qkv(const void* x, const void* w_qkv, int32_t hidden,
                            const cva_kv_cache* cache, const cva_rope_tables* tables,
                            int32_t t0, int32_t k_f, int32_t k_b, void* workspace,
                            size_t ws_bytes, void* out, float* lse, cva_stream_t stream);

/* ---- head-sharded path (several GPUs) -------------------------------------
 * "Accelerating Video Generation Inference with Sequential-Parallel 3D
 * Positional Encoding Using a Global Time Index", section 2A: with the chunk
 * sharded by tokens across G ranks, one all-to-all before the attention
 * hands every rank all tokens of H/G heads, and one after it gives the
 * token slices back. The exchange itself is the caller's collective (NCCL);
 * this is the layout step around it.
 *
 * For i0 < n0 and i1 < n1 copies inner_bytes from src + i0*src_stride0 +
 * i1*src_stride1 to dst + i0*dst_stride0 + i1*dst_stride1 (device memory,
 * byte strides). Every size and stride a multiple of 16 and both pointers
 * 16-byte aligned, else CVA_EINVAL; destination rows must not overlap each
 * other or the source. Swapping the two outer dimensions of an
 * [n0][n1][row] array is (ss0, ss1, ds0, ds1) = (n1*row, row, row, n0*row). */
int cva_copy_rows_2d(const void* src, void* dst, int64_t n0, int64_t n1, int64_t inner_bytes,
                     int64_t src_stride0, int64_t src_stride1, int64_t dst_stride0, int64_t dst_stride1,
                     cva_stream_t stream);

/* The fused chunk call without a caller workspace (the pages have no
 * counterpart; this exists for callers that cannot allocate device memory
 * when they call, such as a plugin whose host runtime owns every allocation
 * and passes it only inputs and outputs, or a loop that forbids allocation
 * after start-up). Same arguments, checks and results as cva_chunk_attention;
 * the scratch is one fixed 64 MiB array inside the library (enough for the
 * 1.3B-shaped 480P chunk at any budget up to 1024 candidate blocks). Shapes and
 * budgets that need more return CVA_ENOMEM without launching. Under CUDA's
 * default lazy module loading the array is reserved on a device by the first
 * call there (which loads the library part that holds it and looks up its
 * address with cudaGetSymbolAddress) and stays reserved until the process
 * exits; that first call can fail for lack of device memory (CVA_ELAUNCH), so
 * make it during start-up, before any stream capture, or set
 * CUDA_MODULE_LOADING=EAGER. Later calls allocate and free nothing. All calls
 * share the one array and keep whatever the last call left in it: calls
 * that overlap on the GPU (different streams, or different host threads on
 * one device) race on it, so order them on one stream. */
int cva_chunk_attention_noalloc(const void* q, const void* k, const void* v,
                                const cva_kv_cache* cache, const cva_rope_tables* tables,
                                int32_t t0, int32_t k_f, int32_t k_b, void* out, float* lse,
                                cva_stream_t stream);

/* Per-stage timing of cva_chunk_attention on this host thread: while set,
 * each call records events[0] before its first launch, events[1] after the
 * rotate/append/pool kernels, events[2] after the selection (right after
 * events[1] when there is none) and events[3] after the attention, all on
 * the call's stream. `events` are cudaEvent_t handles owned by the caller;
 * n must be 4, or 0 with events == NULL to stop. */
int cva_set_stage_events(void* const* events, int32_t n);

/* Diagnostic of the device-side failure path: one CTA waits, through the
 * bounded wait every pipeline role of the kernels uses, on an mbarrier that
 * nothing arrives at, with a limit of limit_us microseconds (1 .. 10^6)
 * instead of the kernels' 4 s. The wait gives up, latches CVA_DEV_TIMEOUT in
 * the device error word (read and cleared by cva_device_status) and raises
 * the CTA's abort flag; result (device, 2 int32) receives {1 if the wait gave
 * up, 1 if the abort flag was raised}. No copy or MMA is in flight, so the
 * kernel returns normally and the context stays usable. */
int cva_diag_wait_timeout(int32_t limit_us, int32_t* result, cva_stream_t stream);

/* Diagnostic of the tensor cores: `ctas` CTAs (at most one per SM) each issue
 * iters x 4 back-to-back tcgen05.mma kind::f16 of shape m x n x 16 (bf16
 * zeros from shared memory, fp32 accumulator in tensor memory) from one
 * thread and wait for them (bounded; a timeout latches CVA_DEV_TIMEOUT);
 * cycles[c] gets CTA c's clock64 span, so cycles / (4 iters) is the time of
 * one MMA. m: 64 or 128; n: a multiple of 8 (m = 64) or 16 (m = 128) in
 * [8, 256]; iters in [1, 65536]. cycles: device buffer of ctas uint64
 * values, 8-byte aligned. It is what shows that a 64-row MMA takes the
 * tensor time of a 128-row one, which is why attention tiles hold 128 rows
 * ("Light Forcing" section 2.2 picks per 64-token query block; two blocks
 * share a tile). */
int cva_diag_mma_cycles(int32_t m, int32_t n, int32_t iters, uint64_t* cycles, int32_t ctas,
                        cva_stream_t stream);

/* Chunk budget from the noise level ("Light Forcing", section 2.1: s_i =
 * s_base - alpha_i beta, alpha_i scaling with the noise level as 1/sqrt(T),
 * beta set so that the total FLOPs meet a target sparsity). Readings: alpha_i
 * = 1/sqrt(i) for chunk i (the noise level grows with the chunk index);
 * density d_i = 1 - s_i clamped to [0, 1] over history blocks; the target is
 * sum_i d_i N_i = (1 - s_target) sum_i N_i over chunks 2..n_chunks, N_i the
 * history blocks of chunk i in a rolling window of `window` frames (chunks
 * of Fc frames, blocks_per_frame blocks); beta by 200 fp64 bisection steps on
 * [-2^20, 2^20]. Writes densities[i - 2] for i = 2..n_chunks (chunk 1 is
 * dense). CVA_EINVAL for n_chunks < 2, Fc < 1, window < Fc, or s outside [0, 1]. */
int cva_cag_noise_densities(int32_t n_chunks, int32_t Fc, int32_t window, int32_t blocks_per_frame,
                            double s_base, double s_target, double* densities);
/* (k_f, k_b) of a chunk at a given density: k_f = min(k_f_max, history),
 * k_b = floor(density * history blocks + 1/2) capped at k_f * blocks. */
int cva_cag_density_budget(int32_t chunk_index, int32_t hist_frames, int32_t blocks_per_frame,
                           int32_t k_f_max, double density, int32_t* k_f, int32_t* k_b);

/* ---- cache arena ---------------------------------------------------------- */

/* Bytes of one layer's cache for `window` frame slots (256-byte aligned parts). */
int cva_kv_cache_bytes(const cva_shape* shape, int32_t window, size_t* bytes);
/* Carves one layer's cache out of caller memory (>= cva_kv_cache_bytes, 256-
 * byte aligned). Does not clear it: slots become valid when appended. */
int cva_kv_cache_init(cva_kv_cache* cache, void* dev_mem, size_t bytes,
                      const cva_shape* shape, int32_t window, int32_t t_begin);

/* ---- chunk budget ("Light Forcing", section 2.1) -------------------------- */

/* (k_f, k_b) of chunk `chunk_index` (1-based) with `hist_frames` history
 * frames of `blocks_per_frame` blocks, in exact integer arithmetic. */
int cva_cag_budget(const cva_cag_cfg* cfg, int32_t chunk_index, int32_t hist_frames,
                   int32_t blocks_per_frame, int32_t* k_f, int32_t* k_b);

#ifdef __cplusplus
}
#endif
#endif /* CVA_H_ */
