// C ABI of libcva: argument checks, workspace and cache layout, and the
// launch sequence of the per-chunk path. Nothing here allocates device
// memory or synchronises (except cva_device_status, which reads the device
// error word).
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "kernels.cuh"

using namespace cva;

namespace {

thread_local char g_msg[512] = "";
thread_local cudaEvent_t g_stage_ev[4] = {nullptr, nullptr, nullptr, nullptr};
thread_local bool g_stage_on = false;

cudaError_t stage_mark(int i, cudaStream_t s) {
  return g_stage_on ? cudaEventRecord(g_stage_ev[i], s) : cudaSuccess;
}

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(CVA_ELAUNCH, "%s: %s", where, cudaGetErrorString(e));
}

// SMs of the current device (cached per device).
static int sm_count() {
  static int counts[128] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 0;
  if (counts[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess) counts[dev] = n;
  }
  return counts[dev];
}

// Device error word, one per device; kernels receive its address.
__device__ int g_dev_err;

int* device_error_word() {
  static std::mutex mu;
  static int* ptrs[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dev_err) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
  }
  return ptrs[dev];
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_shape(const cva_shape* s) {
  if (!s) return fail(CVA_EINVAL, "shape is NULL");
  if (s->batch < 1 || s->heads < 1 || s->frame_h < 1 || s->frame_w < 1 || s->chunk_frames < 1)
    return fail(CVA_EINVAL, "shape: batch, heads, frame_h, frame_w, chunk_frames must be >= 1");
  if (s->head_dim != 64 && s->head_dim != 128)
    return fail(CVA_ENOTSUP, "head_dim %d not supported (64 or 128)", s->head_dim);
  if (s->block != 64 && s->block != 128)
    return fail(CVA_ENOTSUP, "block %d not supported (64 or 128)", s->block);
  if ((int64_t)s->batch * s->heads > 65535) return fail(CVA_ENOTSUP, "batch*heads > 65535");
  const int64_t tf = (int64_t)s->frame_h * s->frame_w;
  if (tf > (1 << 20)) return fail(CVA_ENOTSUP, "tokens per frame > 2^20");
  const Dims d = make_dims(*s);
  if ((int64_t)d.Fc * d.nb > 65535) return fail(CVA_ENOTSUP, "chunk_frames * blocks per frame > 65535");
  return CVA_OK;
}

bool same_shape(const cva_shape& a, const cva_shape& b) {
  return a.batch == b.batch && a.heads == b.heads && a.head_dim == b.head_dim &&
         a.frame_h == b.frame_h && a.frame_w == b.frame_w && a.chunk_frames == b.chunk_frames &&
         a.block == b.block;
}

int check_cache(const cva_kv_cache* c) {
  if (!c) return fail(CVA_EINVAL, "cache is NULL");
  int rc = check_shape(&c->shape);
  if (rc) return rc;
  if (!c->k || !c->v || !c->kpool_blk || !c->kpool_frm)
    return fail(CVA_EINVAL, "cache has a NULL buffer");
  if (!aligned(c->k, 256) || !aligned(c->v, 256) || !aligned(c->kpool_blk, 16) ||
      !aligned(c->kpool_frm, 16))
    return fail(CVA_EINVAL, "cache buffers must be 256-byte (k, v) and 16-byte (pools) aligned");
  if (c->window < c->shape.chunk_frames)
    return fail(CVA_EINVAL, "cache window %d < chunk_frames %d", c->window, c->shape.chunk_frames);
  const Dims d = make_dims(c->shape);
  if ((int64_t)c->window * d.T_pad / 64 >= 65536)
    return fail(CVA_ENOTSUP, "window * padded frame rows too large (>= 2^22 rows)");
  return CVA_OK;
}

int check_tables(const cva_rope_tables* t, const Dims& d, int t0) {
  if (!t) return fail(CVA_EINVAL, "rope tables are NULL");
  if (!t->cos_t || !t->sin_t || !t->cos_h || !t->sin_h || !t->cos_w || !t->sin_w)
    return fail(CVA_EINVAL, "rope tables have a NULL pointer");
  if (t->head_dim != d.D) return fail(CVA_EINVAL, "rope tables built for head_dim %d, shape has %d", t->head_dim, d.D);
  if (t->frame_h < d.Fh || t->frame_w < d.Fw)
    return fail(CVA_ERANGE, "rope tables cover %dx%d positions, frame is %dx%d", t->frame_h, t->frame_w, d.Fh, d.Fw);
  if (t0 < 0 || (int64_t)t0 + d.Fc > t->max_t)
    return fail(CVA_ERANGE, "global time %d..%d outside the temporal table (max_t %d)", t0, t0 + d.Fc - 1, t->max_t);
  if (t->cs_tok && !aligned(t->cs_tok, 16)) return fail(CVA_EINVAL, "cs_tok must be 16-byte aligned");
  return CVA_OK;
}

RopeTab make_tab(const cva_rope_tables* t, int D) {
  RopeTab r;
  r.cos_t = t->cos_t; r.sin_t = t->sin_t; r.cos_h = t->cos_h; r.sin_h = t->sin_h;
  r.cos_w = t->cos_w; r.sin_w = t->sin_w;
  r.cs_tok = t->cs_tok;
  axis_pairs(D, &r.pt, &r.ph, &r.pw);
  r.tab_w = t->frame_w;
  return r;
}

// History frames [t_lo, t_lo + F) a chunk at t0 sees.
void history(const cva_kv_cache* c, int t0, int* t_lo, int* F) {
  int lo = t0 + c->shape.chunk_frames - c->window;
  if (lo < c->t_begin) lo = c->t_begin;
  *t_lo = lo;
  *F = t0 > lo ? t0 - lo : 0;
}

struct ChunkWs {
  size_t q_rot, qpool, frame_idx, block_idx, block_cnt, qpair, attn, total;
};

// Attention scratch: partial (O, max, sum) of the pieces of split tail tiles.
size_t attn_split_bytes(const Dims& d) {
  return round256((size_t)kAttnMaxPieces * 128 * d.D * 4) + round256((size_t)kAttnMaxPieces * 128 * 2 * 4);
}

ChunkWs chunk_ws_layout(const Dims& d, int k_f, int k_b) {
  ChunkWs w;
  const size_t bhq = (size_t)d.B * d.H * d.NQB;
  size_t off = 0;
  w.q_rot = off; off += round256((size_t)d.B * d.H * d.Fc * d.T_pad * d.D * 2);
  w.qpool = off; off += round256(bhq * d.D * 4);
  w.frame_idx = off; off += round256(bhq * (size_t)(k_f > 0 ? k_f : 0) * 4);
  w.block_idx = off; off += round256(bhq * (size_t)(k_b > 0 ? k_b : 0) * 4);
  w.block_cnt = off; off += round256(bhq * 4);
  w.qpair = off; off += round256((size_t)d.B * d.H * ((d.Fc * d.T_pad + 127) / 128) * 2 * 4);
  w.attn = off; off += attn_split_bytes(d);
  w.total = off;
  return w;
}

int check_attn_limits(const Dims& d, int F, bool dense, int k_b_max) {
  const int upb = d.blk / 64;
  const int64_t cur = (int64_t)d.Fc * d.nb * upb;
  int64_t hist;
  if (dense) {
    hist = (int64_t)F * d.nb * upb;
  } else {
    if ((int64_t)F * d.nb > 32 * kAttnMaxBitmapWords)
      return fail(CVA_ENOTSUP, "history blocks %lld exceed %d for the sparse attention",
                  (long long)F * d.nb, 32 * kAttnMaxBitmapWords);
    // a query tile holds nq query blocks (two when blk = 64)
    const int nq = d.blk == 64 ? 2 : 1;
    int64_t u = (int64_t)nq * k_b_max;
    if (u > (int64_t)F * d.nb) u = (int64_t)F * d.nb;
    hist = u * upb;
  }
  // + one padding unit per section
  if (hist + cur + 3 > kAttnMaxEntries)
    return fail(CVA_ENOTSUP, "key units per query tile %lld exceed %d",
                (long long)(hist + cur + 3), kAttnMaxEntries);
  return CVA_OK;
}

}  // namespace

namespace cva {
int report_error(int code, const char* msg) { return fail(code, "%s", msg); }
}  // namespace cva

extern "C" {

int cva_version(void) { return CVA_VERSION; }

const char* cva_last_error(void) { return g_msg; }

int cva_device_status(int32_t* code, int32_t clear) {
  if (!code) return fail(CVA_EINVAL, "code is NULL");
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_dev_err, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  *code = v;
  if (clear) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_dev_err, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
  }
  return CVA_OK;
}

int cva_set_stage_events(void* const* events, int32_t n) {
  if (n == 0 && events == nullptr) {
    g_stage_on = false;
    return CVA_OK;
  }
  if (n != 4 || !events) return fail(CVA_EINVAL, "stage events: pass 4 events, or NULL and 0");
  for (int i = 0; i < 4; ++i) {
    if (!events[i]) return fail(CVA_EINVAL, "stage event %d is NULL", i);
    g_stage_ev[i] = static_cast<cudaEvent_t>(events[i]);
  }
  g_stage_on = true;
  return CVA_OK;
}

int cva_diag_wait_timeout(int32_t limit_us, int32_t* result, cva_stream_t stream) {
  if (!result) return fail(CVA_EINVAL, "result is NULL");
  if (!aligned(result, 4)) return fail(CVA_EINVAL, "result must be 4-byte aligned");
  if (limit_us < 1 || limit_us > 1000000) return fail(CVA_EINVAL, "limit_us must lie in [1, 1000000]");
  int* err = device_error_word();
  if (!err) return fail(CVA_ELAUNCH, "device error word unavailable");
  cudaError_t e = launch_wait_timeout(err, result, (uint64_t)limit_us * 1000ull, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CVA_OK : cuda_fail(e, "diag_wait_timeout launch");
}

int cva_diag_mma_cycles(int32_t m, int32_t n, int32_t iters, uint64_t* cycles, int32_t ctas,
                        cva_stream_t stream) {
  if (!cycles) return fail(CVA_EINVAL, "cycles is NULL");
  if (!aligned(cycles, 8)) return fail(CVA_EINVAL, "cycles must be 8-byte aligned");
  if (m != 64 && m != 128) return fail(CVA_EINVAL, "m must be 64 or 128");
  if (n < 8 || n > 256 || n % (m == 64 ? 8 : 16)) return fail(CVA_EINVAL, "n must be a multiple of %d in [8, 256]", m == 64 ? 8 : 16);
  if (iters < 1 || iters > 65536) return fail(CVA_EINVAL, "iters must lie in [1, 65536]");
  const int nsm = sm_count();
  if (ctas < 1 || (nsm > 0 && ctas > nsm)) return fail(CVA_EINVAL, "ctas must lie in [1, SM count]");
  int* err = device_error_word();
  if (!err) return fail(CVA_ELAUNCH, "device error word unavailable");
  cudaError_t e = launch_mma_cycles(m, n, iters, reinterpret_cast<unsigned long long*>(cycles), ctas, err,
                                    static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CVA_OK : cuda_fail(e, "diag_mma_cycles launch");
}

int cva_rope_axis_pairs(int32_t head_dim, int32_t* p_t, int32_t* p_h, int32_t* p_w) {
  if (!p_t || !p_h || !p_w) return fail(CVA_EINVAL, "NULL output");
  if (head_dim < 6 || head_dim % 2) return fail(CVA_EINVAL, "head_dim must be even and >= 6");
  int a, b, c;
  axis_pairs(head_dim, &a, &b, &c);
  *p_t = a; *p_h = b; *p_w = c;
  return CVA_OK;
}

int cva_rope3d_precompute(const cva_rope_cfg* cfg, float* cos_t, float* sin_t, float* cos_h,
                          float* sin_h, float* cos_w, float* sin_w) {
  if (!cfg) return fail(CVA_EINVAL, "cfg is NULL");
  if (!cos_t || !sin_t || !cos_h || !sin_h || !cos_w || !sin_w) return fail(CVA_EINVAL, "NULL table");
  if (cfg->head_dim < 6 || cfg->head_dim % 2) return fail(CVA_EINVAL, "head_dim must be even and >= 6");
  if (cfg->max_t < 1 || cfg->frame_h < 1 || cfg->frame_w < 1) return fail(CVA_EINVAL, "table rows must be >= 1");
  if (!(cfg->theta > 1.0)) return fail(CVA_EINVAL, "theta must be > 1");
  int p[3];
  axis_pairs(cfg->head_dim, &p[0], &p[1], &p[2]);
  const int rows[3] = {cfg->max_t, cfg->frame_h, cfg->frame_w};
  float* cs[3] = {cos_t, cos_h, cos_w};
  float* sn[3] = {sin_t, sin_h, sin_w};
  for (int a = 0; a < 3; ++a) {
    for (int pos = 0; pos < rows[a]; ++pos) {
      for (int j = 0; j < p[a]; ++j) {
        // rate theta^(-2j / (2 p_a)) radians per unit of position
        const double rate = pow(cfg->theta, -(2.0 * j) / (2.0 * p[a]));
        const double ang = (double)pos * rate;
        cs[a][(size_t)pos * p[a] + j] = (float)cos(ang);
        sn[a][(size_t)pos * p[a] + j] = (float)sin(ang);
      }
    }
  }
  return CVA_OK;
}

int cva_rope3d_precompute_tokens(const cva_rope_cfg* cfg, float* cs_tok) {
  if (!cfg || !cs_tok) return fail(CVA_EINVAL, "NULL argument");
  if (cfg->head_dim < 6 || cfg->head_dim % 2) return fail(CVA_EINVAL, "head_dim must be even and >= 6");
  if (cfg->frame_h < 1 || cfg->frame_w < 1) return fail(CVA_EINVAL, "table rows must be >= 1");
  if (!(cfg->theta > 1.0)) return fail(CVA_EINVAL, "theta must be > 1");
  int pt, ph, pw;
  axis_pairs(cfg->head_dim, &pt, &ph, &pw);
  const int np = cfg->head_dim / 2;
  // the same values as the per-axis tables: (float)cos/sin of pos * rate in double
  for (int h = 0; h < cfg->frame_h; ++h) {
    for (int w = 0; w < cfg->frame_w; ++w) {
      float* e = cs_tok + ((size_t)h * cfg->frame_w + w) * np * 2;
      for (int p = 0; p < np; ++p) {
        int pos = 0, j = 0, pa = 1;
        if (p < pt) {
          e[2 * p] = 1.f;
          e[2 * p + 1] = 0.f;
          continue;
        } else if (p < pt + ph) {
          pos = h; j = p - pt; pa = ph;
        } else {
          pos = w; j = p - pt - ph; pa = pw;
        }
        const double rate = pow(cfg->theta, -(2.0 * j) / (2.0 * pa));
        const double ang = (double)pos * rate;
        e[2 * p] = (float)cos(ang);
        e[2 * p + 1] = (float)sin(ang);
      }
    }
  }
  return CVA_OK;
}

int cva_history_frames(const cva_kv_cache* cache, int32_t t0, int32_t* t_lo, int32_t* count) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (!t_lo || !count) return fail(CVA_EINVAL, "NULL output");
  if (t0 < cache->t_begin) return fail(CVA_ERANGE, "t0 %d before the stream start %d", t0, cache->t_begin);
  int lo, F;
  history(cache, t0, &lo, &F);
  *t_lo = lo;
  *count = F;
  return CVA_OK;
}

int cva_kv_cache_bytes(const cva_shape* shape, int32_t window, size_t* bytes) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!bytes) return fail(CVA_EINVAL, "bytes is NULL");
  if (window < shape->chunk_frames) return fail(CVA_EINVAL, "window < chunk_frames");
  const Dims d = make_dims(*shape);
  const size_t slots = (size_t)d.B * d.H * window;
  *bytes = 2 * round256(slots * d.T_pad * d.D * 2) + round256(slots * d.nb * d.D * 4) +
           round256(slots * d.D * 4);
  return CVA_OK;
}

int cva_kv_cache_init(cva_kv_cache* cache, void* dev_mem, size_t bytes, const cva_shape* shape,
                      int32_t window, int32_t t_begin) {
  if (!cache || !dev_mem) return fail(CVA_EINVAL, "NULL cache or memory");
  size_t need = 0;
  int rc = cva_kv_cache_bytes(shape, window, &need);
  if (rc) return rc;
  if (bytes < need) return fail(CVA_ENOMEM, "cache arena %zu bytes < %zu needed", bytes, need);
  if (!aligned(dev_mem, 256)) return fail(CVA_EINVAL, "cache arena must be 256-byte aligned");
  if (t_begin < 0) return fail(CVA_EINVAL, "t_begin < 0");
  const Dims d = make_dims(*shape);
  const size_t slots = (size_t)d.B * d.H * window;
  char* p = static_cast<char*>(dev_mem);
  cache->k = p; p += round256(slots * d.T_pad * d.D * 2);
  cache->v = p; p += round256(slots * d.T_pad * d.D * 2);
  cache->kpool_blk = reinterpret_cast<float*>(p); p += round256(slots * d.nb * d.D * 4);
  cache->kpool_frm = reinterpret_cast<float*>(p);
  cache->window = window;
  cache->t_begin = t_begin;
  cache->shape = *shape;
  return check_cache(cache);
}

int cva_cag_budget(const cva_cag_cfg* cfg, int32_t chunk_index, int32_t hist_frames,
                   int32_t blocks_per_frame, int32_t* k_f, int32_t* k_b) {
  if (!cfg || !k_f || !k_b) return fail(CVA_EINVAL, "NULL argument");
  if (chunk_index < 1 || hist_frames < 0 || blocks_per_frame < 1)
    return fail(CVA_EINVAL, "chunk_index >= 1, hist_frames >= 0, blocks_per_frame >= 1 required");
  const int64_t all = (int64_t)hist_frames * blocks_per_frame;
  if (cfg->dense || chunk_index <= 1 || hist_frames == 0) {
    *k_f = hist_frames;
    *k_b = (int32_t)all;
    return CVA_OK;
  }
  if (cfg->k_f_max < 1) return fail(CVA_EINVAL, "k_f_max must be >= 1");
  const int kf = cfg->k_f_max < hist_frames ? cfg->k_f_max : hist_frames;
  const int64_t cand = (int64_t)kf * blocks_per_frame;
  int64_t kb;
  if (cfg->k_b_fixed >= 0) {
    kb = cfg->k_b_fixed;
  } else {
    if (cfg->d_base_den <= 0 || cfg->d_slope_den <= 0) return fail(CVA_EINVAL, "denominators must be > 0");
    // d = d_base + d_slope * (i - pivot) as one fraction num/den (exact)
    const int64_t den = cfg->d_base_den * cfg->d_slope_den;
    int64_t num = cfg->d_base_num * cfg->d_slope_den +
                  cfg->d_slope_num * cfg->d_base_den * (int64_t)(chunk_index - cfg->pivot);
    if (num < 0) num = 0;
    if (num > den) num = den;
    // floor(d * all + 1/2) = floor((2 * num * all + den) / (2 * den))
    kb = (2 * num * all + den) / (2 * den);
  }
  if (kb > cand) kb = cand;
  *k_f = kf;
  *k_b = (int32_t)kb;
  return CVA_OK;
}

int cva_rope3d_apply(const void* x, void* y, const cva_rope_tables* tables, const cva_shape* shape,
                     int32_t t0, int32_t out_layout, cva_stream_t stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!x || !y) return fail(CVA_EINVAL, "x or y is NULL");
  if (!aligned(x, 16) || !aligned(y, 16)) return fail(CVA_EINVAL, "x and y must be 16-byte aligned");
  if (out_layout != 0 && out_layout != 1) return fail(CVA_EINVAL, "out_layout must be 0 or 1");
  const Dims d = make_dims(*shape);
  rc = check_tables(tables, d, t0);
  if (rc) return rc;
  RopePoolArgs a = {};
  a.job[0] = {static_cast<const uint16_t*>(x), kTokenMajor, static_cast<uint16_t*>(y),
              out_layout == 0 ? (int)kTokenMajor : (int)kHeadMajor, 1, nullptr, kPoolNone};
  a.njobs = 1;
  a.err = device_error_word();
  a.tab = make_tab(tables, d.D);
  a.d = d;
  a.t0 = t0;
  a.W = 1;
  cudaError_t e = launch_rope_pool(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CVA_OK : cuda_fail(e, "rope3d_apply launch");
}

int cva_kv_append(const void* k, const void* v, const cva_kv_cache* cache,
                  const cva_rope_tables* tables, int32_t t0, cva_stream_t stream) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (!k || !v) return fail(CVA_EINVAL, "k or v is NULL");
  if (!aligned(k, 16) || !aligned(v, 16)) return fail(CVA_EINVAL, "k and v must be 16-byte aligned");
  const Dims d = make_dims(cache->shape);
  if (t0 < cache->t_begin) return fail(CVA_ERANGE, "t0 %d before the stream start %d", t0, cache->t_begin);
  if (tables) {
    rc = check_tables(tables, d, t0);
    if (rc) return rc;
  }
  RopePoolArgs a = {};
  a.job[0] = {static_cast<const uint16_t*>(k), kTokenMajor, static_cast<uint16_t*>(cache->k),
              kCacheSlots, tables ? 1 : 0, cache->kpool_blk, kPoolCache};
  a.job[1] = {static_cast<const uint16_t*>(v), kTokenMajor, static_cast<uint16_t*>(cache->v),
              kCacheSlots, 0, nullptr, kPoolNone};
  a.njobs = 2;
  a.err = device_error_word();
  if (tables) a.tab = make_tab(tables, d.D);
  else axis_pairs(d.D, &a.tab.pt, &a.tab.ph, &a.tab.pw);
  a.d = d;
  a.t0 = t0;
  a.W = cache->window;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_rope_pool(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "kv_append launch");
  FramePoolArgs fp = {cache->kpool_blk, cache->kpool_frm, kPoolCache, d, t0, cache->window};
  e = launch_frame_pool(fp, s);
  return e == cudaSuccess ? CVA_OK : cuda_fail(e, "kv_append frame pool launch");
}

}  // extern "C"

// The fused projection; with frame_pool the frame means of the new cache
// frames follow in a second launch (the fused chunk call has the attention
// launch compute them instead).
static int qkv_rope_append_impl(const void* x, const void* w_qkv, int32_t hidden, const cva_kv_cache* cache,
                                const cva_rope_tables* tables, int32_t t0, void* q_rot, float* qpool_blk,
                                cva_stream_t stream, bool frame_pool) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (!x || !w_qkv || !q_rot || !tables) return fail(CVA_EINVAL, "x, w_qkv, q_rot or tables is NULL");
  if (!aligned(x, 16) || !aligned(w_qkv, 16) || !aligned(q_rot, 16))
    return fail(CVA_EINVAL, "x, w_qkv and q_rot must be 16-byte aligned");
  if (hidden < 64 || hidden % 64) return fail(CVA_ENOTSUP, "hidden %d must be a positive multiple of 64", hidden);
  const Dims d = make_dims(cache->shape);
  if (t0 < cache->t_begin) return fail(CVA_ERANGE, "t0 %d before the stream start %d", t0, cache->t_begin);
  rc = check_tables(tables, d, t0);
  if (rc) return rc;
  QkvArgs a = {};
  a.d = d;
  a.C = hidden;
  a.t0 = t0;
  a.W = cache->window;
  a.tab = make_tab(tables, d.D);
  a.q_rot = static_cast<uint16_t*>(q_rot);
  a.k_cache = static_cast<uint16_t*>(cache->k);
  a.v_cache = static_cast<uint16_t*>(cache->v);
  a.qpool = qpool_blk;
  a.kpool_blk = cache->kpool_blk;
  a.MT = (d.Fc * d.T_pad + 127) / 128;
  a.NT = (3 * d.H * d.D + 255) / 256;
  a.err = device_error_word();
  if (a.MT > 65535) return fail(CVA_ENOTSUP, "padded chunk rows %d too many", d.Fc * d.T_pad);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const char* why = "";
  cudaError_t e = launch_qkv_rope(a, x, w_qkv, s, &why);
  if (e == cudaErrorInvalidValue && why[0]) return fail(CVA_ELAUNCH, "qkv_rope_append: %s", why);
  if (e != cudaSuccess) return cuda_fail(e, "qkv_rope_append launch");
  if (!frame_pool) return CVA_OK;
  FramePoolArgs fp = {cache->kpool_blk, cache->kpool_frm, kPoolCache, d, t0, cache->window};
  e = launch_frame_pool(fp, s);
  return e == cudaSuccess ? CVA_OK : cuda_fail(e, "qkv_rope_append frame pool launch");
}

extern "C" {

int cva_qkv_rope_append(const void* x, const void* w_qkv, int32_t hidden, const cva_kv_cache* cache,
                        const cva_rope_tables* tables, int32_t t0, void* q_rot, float* qpool_blk,
                        cva_stream_t stream) {
  return qkv_rope_append_impl(x, w_qkv, hidden, cache, tables, t0, q_rot, qpool_blk, stream, true);
}

int cva_hsa_compress(const void* q_rot, const cva_shape* shape, float* qpool_blk, float* qpool_frm,
                     cva_stream_t stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!q_rot || !qpool_blk) return fail(CVA_EINVAL, "q_rot or qpool_blk is NULL");
  if (!aligned(q_rot, 16)) return fail(CVA_EINVAL, "q_rot must be 16-byte aligned");
  const Dims d = make_dims(*shape);
  RopePoolArgs a = {};
  a.job[0] = {static_cast<const uint16_t*>(q_rot), kHeadMajor, nullptr, kHeadMajor, 0, qpool_blk,
              kPoolChunk};
  a.njobs = 1;
  a.err = device_error_word();
  axis_pairs(d.D, &a.tab.pt, &a.tab.ph, &a.tab.pw);
  a.d = d;
  a.t0 = 0;
  a.W = 1;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_rope_pool(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "hsa_compress launch");
  if (qpool_frm) {
    FramePoolArgs fp = {qpool_blk, qpool_frm, kPoolChunk, d, 0, 1};
    e = launch_frame_pool(fp, s);
    if (e != cudaSuccess) return cuda_fail(e, "hsa_compress frame pool launch");
  }
  return CVA_OK;
}

// Arguments of the rotate/append/pool launch of steps 1-3: Q rotated into
// q_rot (head-major, frames padded to whole blocks) with its block means in
// qpool (when not NULL), K rotated and V copied into the cache slots of the
// chunk's frames with the block means of the stored keys.
static RopePoolArgs chunk_rope_args(const void* q, const void* k, const void* v, const cva_kv_cache* cache,
                                    const cva_rope_tables* tables, int32_t t0, uint16_t* q_rot,
                                    float* qpool) {
  const Dims d = make_dims(cache->shape);
  RopePoolArgs a = {};
  a.job[0] = {static_cast<const uint16_t*>(q), kTokenMajor, q_rot, kHeadMajor, 1, qpool,
              qpool ? (int)kPoolChunk : (int)kPoolNone};
  a.job[1] = {static_cast<const uint16_t*>(k), kTokenMajor, static_cast<uint16_t*>(cache->k),
              kCacheSlots, 1, cache->kpool_blk, kPoolCache};
  a.job[2] = {static_cast<const uint16_t*>(v), kTokenMajor, static_cast<uint16_t*>(cache->v),
              kCacheSlots, 0, nullptr, kPoolNone};
  a.njobs = 3;
  a.err = device_error_word();
  a.tab = make_tab(tables, d.D);
  a.d = d;
  a.t0 = t0;
  a.W = cache->window;
  return a;
}

// Selection launch; topp > 0 switches the second level to the top-p budget
// with cap k_b.
// dependent: the launch directly follows the chunk's rotation kernel on the
// stream (programmatic dependent launch).
static int select_impl(const float* qpool_blk, const cva_kv_cache* cache, int t0, int k_f, int k_b,
                       int32_t* frame_idx, int32_t* block_idx, int32_t* block_cnt, int k_b_max,
                       float topp, cudaStream_t s, bool dependent = false) {
  const Dims d = make_dims(cache->shape);
  int t_lo, F;
  history(cache, t0, &t_lo, &F);
  const int kfe = k_f < F ? k_f : F;
  if (F > 0 && k_f < 1) return fail(CVA_ERANGE, "k_f must be >= 1 when there is history");
  if (k_b < 0 || (int64_t)k_b > (int64_t)kfe * d.nb)
    return fail(CVA_ERANGE, "k_b %d outside [0, %d] (k_f_eff * blocks per frame)", k_b, kfe * d.nb);
  if (F > 256) return fail(CVA_ENOTSUP, "history frames %d > 256", F);
  if ((int64_t)kfe * d.nb > 1024) return fail(CVA_ENOTSUP, "candidate blocks %d > 1024", kfe * d.nb);
  SelectArgs a = {};
  a.qpool = qpool_blk;
  a.kpool_blk = cache->kpool_blk;
  a.kpool_frm = cache->kpool_frm;
  a.frame_idx = frame_idx;
  a.block_idx = block_idx;
  a.block_cnt = block_cnt;
  a.d = d;
  a.W = cache->window;
  a.t_lo = t_lo;
  a.F = F;
  a.k_f = kfe;
  a.k_b = k_b;
  a.k_f_stride = kfe;
  a.k_b_max = k_b_max;
  a.topp = topp;
  a.temp_log2 = (float)(1.4426950408889634 / sqrt((double)d.D));
  if (F == 0) {
    // Nothing to pick: every count is zero.
    if (block_cnt) {
      cudaError_t e = cudaMemsetAsync(block_cnt, 0, (size_t)d.B * d.H * d.NQB * 4, s);
      if (e != cudaSuccess) return cuda_fail(e, "hsa_select memset");
    }
    return CVA_OK;
  }
  cudaError_t e = launch_select(a, s, dependent);
  return e == cudaSuccess ? CVA_OK : cuda_fail(e, "hsa_select launch");
}

int cva_hsa_select(const float* qpool_blk, const cva_kv_cache* cache, int32_t t0, int32_t k_f,
                   int32_t k_b, int32_t* frame_idx, int32_t* block_idx, int32_t* block_cnt,
                   cva_stream_t stream) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (!qpool_blk || !block_idx || !block_cnt) return fail(CVA_EINVAL, "NULL buffer");
  if (t0 < cache->t_begin) return fail(CVA_ERANGE, "t0 %d before the stream start %d", t0, cache->t_begin);
  return select_impl(qpool_blk, cache, t0, k_f, k_b, frame_idx, block_idx, block_cnt, k_b, 0.f,
                     static_cast<cudaStream_t>(stream));
}

static bool topp_ok(float p) { return p > 0.f && p <= 1.f; }

int cva_hsa_select_topp(const float* qpool_blk, const cva_kv_cache* cache, int32_t t0, int32_t k_f,
                        int32_t k_cap, float p, int32_t* frame_idx, int32_t* block_idx,
                        int32_t* block_cnt, cva_stream_t stream) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (!qpool_blk || !block_idx || !block_cnt) return fail(CVA_EINVAL, "NULL buffer");
  if (!topp_ok(p)) return fail(CVA_ERANGE, "p must lie in (0, 1]");
  if (k_cap < 1) return fail(CVA_ERANGE, "k_cap must be >= 1");
  if (t0 < cache->t_begin) return fail(CVA_ERANGE, "t0 %d before the stream start %d", t0, cache->t_begin);
  return select_impl(qpool_blk, cache, t0, k_f, k_cap, frame_idx, block_idx, block_cnt, k_cap, p,
                     static_cast<cudaStream_t>(stream));
}

int cva_attn_workspace_bytes(const cva_shape* shape, int32_t k_b_max, size_t* bytes) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!bytes) return fail(CVA_EINVAL, "bytes is NULL");
  (void)k_b_max;
  *bytes = attn_split_bytes(make_dims(*shape));
  return CVA_OK;
}

// Tiles of two 64-row query blocks paired by their picked frames (the fused
// calls with a selection); *qpair stays NULL when blocks are 128 rows (one
// block per tile), when fewer than 2 k_f history frames leave little to pair,
// or beyond the pairing's limits (tiles then hold blocks 2m and 2m+1).
static int pair_impl(const Dims& d, const cva_kv_cache* cache, int t0, int k_f, const int32_t* fidx,
                     int32_t* qpair_ws, const int32_t** qpair, cudaStream_t s, bool dependent) {
  *qpair = nullptr;
  if (d.blk != 64) return CVA_OK;
  int t_lo, F;
  history(cache, t0, &t_lo, &F);
  const int kfe = k_f < F ? k_f : F;
  // Pairs pay off only when the query blocks' frame picks can differ much:
  // with at least twice as many history frames as picks.
  if (F == 0 || kfe < 1 || F < 2 * kfe) return CVA_OK;
  const int MT = (d.Fc * d.T_pad + 127) / 128;
  cudaError_t e = launch_pair_query_blocks(fidx, kfe, d, t_lo, F, MT, qpair_ws, s, dependent);
  if (e == cudaErrorInvalidValue) return CVA_OK;  // beyond the pairing's limits: default tiles
  if (e != cudaSuccess) return cuda_fail(e, "pair_query_blocks launch");
  *qpair = qpair_ws;
  return CVA_OK;
}

// frame_means: the launch also writes the frame means of the chunk's cache
// frames (its spare warps), from the block means the chunk's append wrote.
static int attn_impl(const void* q_rot, const cva_kv_cache* cache, int t0, const int32_t* block_idx,
                     const int32_t* block_cnt, int k_b_max, void* out, float* lse, void* split_ws,
                     size_t split_bytes, cudaStream_t s, bool frame_means = false,
                     const int32_t* qpair = nullptr, bool dependent = false) {
  const Dims d = make_dims(cache->shape);
  int t_lo, F;
  history(cache, t0, &t_lo, &F);
  int rc = check_attn_limits(d, F, block_idx == nullptr, k_b_max);
  if (rc) return rc;
  AttnArgs a = {};
  a.block_idx = block_idx;
  a.block_cnt = block_cnt;
  a.k_b_max = k_b_max;
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  a.err = device_error_word();
  a.d = d;
  a.W = cache->window;
  a.t0 = t0;
  a.t_lo = t_lo;
  a.F = F;
  a.MT = (d.Fc * d.T_pad + 127) / 128;
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)d.D));
  if (frame_means) {
    a.kpool_blk = cache->kpool_blk;
    a.kpool_frm = cache->kpool_frm;
  }
  a.qpair = qpair;
  // Tail split: the tiles of the last, partial wave are cut into key-range
  // pieces so that they fill the SMs (needs the scratch; else unsplit).
  const int tiles = a.MT * d.B * d.H;
  a.Qf = tiles;
  a.pieces = 1;
  const int nsm = sm_count();
  if (split_ws && split_bytes >= attn_split_bytes(d) && nsm > 0) {
    const int tail = tiles % nsm;
    int pieces = tail > 0 ? nsm / tail : 0;
    if (tail > 0 && pieces > kAttnMaxPieces / tail) pieces = kAttnMaxPieces / tail;
    if (pieces >= 2) {
      a.Qf = tiles - tail;
      a.pieces = pieces;
      a.part_o = static_cast<float*>(split_ws);
      a.part_ml = reinterpret_cast<float*>(static_cast<char*>(split_ws) +
                                           round256((size_t)kAttnMaxPieces * 128 * d.D * 4));
    }
  }
  const char* why = "";
  cudaError_t e = launch_attention(a, q_rot, cache->k, cache->v, s, &why, dependent);
  if (e == cudaErrorInvalidValue && why[0]) return fail(CVA_ELAUNCH, "attention: %s", why);
  return e == cudaSuccess ? CVA_OK : cuda_fail(e, "blocksparse_attn_fwd launch");
}

int cva_blocksparse_attn_fwd(const void* q_rot, const cva_kv_cache* cache, int32_t t0,
                             const int32_t* block_idx, const int32_t* block_cnt, int32_t k_b_max,
                             void* out, float* lse, void* workspace, size_t ws_bytes,
                             cva_stream_t stream) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (!q_rot || !out) return fail(CVA_EINVAL, "q_rot or out is NULL");
  if (!aligned(q_rot, 16) || !aligned(out, 16)) return fail(CVA_EINVAL, "q_rot and out must be 16-byte aligned");
  if (t0 < cache->t_begin) return fail(CVA_ERANGE, "t0 %d before the stream start %d", t0, cache->t_begin);
  if (block_idx && (!block_cnt || k_b_max < 0)) return fail(CVA_EINVAL, "sparse call needs block_cnt and k_b_max >= 0");
  if (workspace && !aligned(workspace, 256)) return fail(CVA_EINVAL, "workspace must be 256-byte aligned");
  return attn_impl(q_rot, cache, t0, block_idx, block_cnt, block_idx ? k_b_max : 0, out, lse,
                   workspace, workspace ? ws_bytes : 0, static_cast<cudaStream_t>(stream));
}

int cva_chunk_attention_qkv(const void* x, const void* w_qkv, int32_t hidden, const cva_kv_cache* cache,
                            const cva_rope_tables* tables, int32_t t0, int32_t k_f, int32_t k_b,
                            void* workspace, size_t ws_bytes, void* out, float* lse, cva_stream_t stream) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (!out || !workspace) return fail(CVA_EINVAL, "NULL buffer");
  if (!aligned(out, 16) || !aligned(workspace, 256))
    return fail(CVA_EINVAL, "out must be 16-byte and workspace 256-byte aligned");
  const Dims d = make_dims(cache->shape);
  const bool dense = k_f < 0;
  const ChunkWs w = chunk_ws_layout(d, dense ? 0 : k_f, dense ? 0 : k_b);
  if (ws_bytes < w.total) return fail(CVA_ENOMEM, "workspace %zu bytes < %zu needed", ws_bytes, w.total);
  if (t0 < cache->t_begin) return fail(CVA_ERANGE, "t0 %d before the stream start %d", t0, cache->t_begin);
  int t_lo, F;
  history(cache, t0, &t_lo, &F);
  if (!dense) {
    const int kfe = k_f < F ? k_f : F;
    if (F > 0 && k_f < 1) return fail(CVA_ERANGE, "k_f must be >= 1 when there is history");
    if (k_b < 0 || (int64_t)k_b > (int64_t)kfe * d.nb)
      return fail(CVA_ERANGE, "k_b %d outside [0, %d] (k_f_eff * blocks per frame)", k_b, kfe * d.nb);
    if (F > 256) return fail(CVA_ENOTSUP, "history frames %d > 256", F);
    if ((int64_t)kfe * d.nb > 1024) return fail(CVA_ENOTSUP, "candidate blocks %d > 1024", kfe * d.nb);
  }
  rc = check_attn_limits(d, F, dense || F == 0, dense ? 0 : k_b);
  if (rc) return rc;
  char* ws = static_cast<char*>(workspace);
  uint16_t* q_rot = reinterpret_cast<uint16_t*>(ws + w.q_rot);
  float* qpool = reinterpret_cast<float*>(ws + w.qpool);
  int32_t* fidx = reinterpret_cast<int32_t*>(ws + w.frame_idx);
  int32_t* bidx = reinterpret_cast<int32_t*>(ws + w.block_idx);
  int32_t* bcnt = reinterpret_cast<int32_t*>(ws + w.block_cnt);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool sparse = !dense && F > 0;
  // Each kernel after the first one follows one of this call's kernels:
  // programmatic dependent launches, unless stage events sit between them.
  const bool chain = !g_stage_on;
  cudaError_t e = stage_mark(0, s);
  if (e != cudaSuccess) return cuda_fail(e, "stage event");
  // steps 1-3: projection, rotation, append and pooling in the fused kernel
  rc = qkv_rope_append_impl(x, w_qkv, hidden, cache, tables, t0, q_rot, sparse ? qpool : nullptr, stream, false);
  if (rc) return rc;
  if ((e = stage_mark(1, s)) != cudaSuccess) return cuda_fail(e, "stage event");
  const int32_t* qpair = nullptr;
  if (sparse) {
    rc = select_impl(qpool, cache, t0, k_f, k_b, fidx, bidx, bcnt, k_b, 0.f, s, chain);
    if (rc) return rc;
    rc = pair_impl(d, cache, t0, k_f, fidx, reinterpret_cast<int32_t*>(ws + w.qpair), &qpair, s, chain);
    if (rc) return rc;
  }
  if ((e = stage_mark(2, s)) != cudaSuccess) return cuda_fail(e, "stage event");
  rc = attn_impl(q_rot, cache, t0, sparse ? bidx : nullptr, sparse ? bcnt : nullptr,
                 sparse ? k_b : 0, out, lse, ws + w.attn, attn_split_bytes(d), s, true, qpair, chain);
  if (rc) return rc;
  if ((e = stage_mark(3, s)) != cudaSuccess) return cuda_fail(e, "stage event");
  return CVA_OK;
}

int cva_rotate_append_pool(const void* q, const void* k, const void* v, const cva_kv_cache* cache,
                           const cva_rope_tables* tables, int32_t t0, void* q_rot, float* qpool_blk,
                           cva_stream_t stream) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (!q || !k || !v || !q_rot) return fail(CVA_EINVAL, "NULL buffer");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(q_rot, 16))
    return fail(CVA_EINVAL, "q, k, v and q_rot must be 16-byte aligned");
  if (qpool_blk && !aligned(qpool_blk, 16)) return fail(CVA_EINVAL, "qpool_blk must be 16-byte aligned");
  if (t0 < cache->t_begin) return fail(CVA_ERANGE, "t0 %d before the stream start %d", t0, cache->t_begin);
  const Dims d = make_dims(cache->shape);
  rc = check_tables(tables, d, t0);
  if (rc) return rc;
  const RopePoolArgs a = chunk_rope_args(q, k, v, cache, tables, t0, static_cast<uint16_t*>(q_rot), qpool_blk);
  cudaError_t e = launch_rope_pool(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CVA_OK : cuda_fail(e, "rotate_append_pool launch");
}

int cva_kv_frame_means(const cva_kv_cache* cache, int32_t t0, cva_stream_t stream) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (t0 < cache->t_begin) return fail(CVA_ERANGE, "t0 %d before the stream start %d", t0, cache->t_begin);
  const Dims d = make_dims(cache->shape);
  FramePoolArgs fp = {cache->kpool_blk, cache->kpool_frm, kPoolCache, d, t0, cache->window};
  cudaError_t e = launch_frame_pool(fp, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CVA_OK : cuda_fail(e, "kv_frame_means launch");
}

int cva_copy_rows_2d(const void* src, void* dst, int64_t n0, int64_t n1, int64_t inner_bytes,
                     int64_t src_stride0, int64_t src_stride1, int64_t dst_stride0, int64_t dst_stride1,
                     cva_stream_t stream) {
  if (n0 < 0 || n1 < 0 || inner_bytes < 0) return fail(CVA_EINVAL, "negative size");
  if (n0 == 0 || n1 == 0 || inner_bytes == 0) return CVA_OK;
  if (!src || !dst) return fail(CVA_EINVAL, "NULL buffer");
  const int64_t v[5] = {inner_bytes, src_stride0, src_stride1, dst_stride0, dst_stride1};
  for (int i = 0; i < 5; ++i)
    if (v[i] % 16) return fail(CVA_EINVAL, "sizes and strides must be multiples of 16 bytes");
  if (!aligned(src, 16) || !aligned(dst, 16)) return fail(CVA_EINVAL, "src and dst must be 16-byte aligned");
  RowCopy2D c = {n0, n1, inner_bytes, src_stride0, src_stride1, dst_stride0, dst_stride1};
  cudaError_t e = launch_copy_rows_2d(src, dst, c, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CVA_OK : cuda_fail(e, "copy_rows_2d launch");
}

int cva_cag_noise_densities(int32_t n_chunks, int32_t Fc, int32_t window, int32_t blocks_per_frame,
                            double s_base, double s_target, double* densities) {
  if (!densities) return fail(CVA_EINVAL, "densities is NULL");
  if (n_chunks < 2 || Fc < 1 || window < Fc || blocks_per_frame < 1)
    return fail(CVA_EINVAL, "n_chunks >= 2, Fc >= 1, window >= Fc and blocks_per_frame >= 1 required");
  if (!(s_base >= 0.0 && s_base <= 1.0 && s_target >= 0.0 && s_target <= 1.0))
    return fail(CVA_EINVAL, "sparsities must lie in [0, 1]");
  // Same fp64 operations, in the same order, as the reference statement.
  const int n = n_chunks - 1;  // chunks 2..n_chunks
  auto N = [&](int i) { int f = Fc * (i - 1); if (f > window - Fc) f = window - Fc; return (double)f * blocks_per_frame; };
  auto alpha = [&](int i) { return 1.0 / sqrt((double)i); };
  const double d0 = 1.0 - s_base;
  double nsum = 0.0;
  for (int i = 2; i <= n_chunks; ++i) nsum += N(i);
  const double goal = (1.0 - s_target) * nsum;
  auto dens = [&](int i, double beta) {
    double v = d0 + alpha(i) * beta;
    if (v < 0.0) v = 0.0;
    if (v > 1.0) v = 1.0;
    return v;
  };
  auto total = [&](double beta) {
    double s = 0.0;
    for (int i = 2; i <= n_chunks; ++i) s += dens(i, beta) * N(i);
    return s;
  };
  double lo = -1048576.0, hi = 1048576.0;
  for (int it = 0; it < 200; ++it) {
    const double mid = 0.5 * (lo + hi);
    if (total(mid) < goal) lo = mid;
    else hi = mid;
  }
  for (int k = 0; k < n; ++k) densities[k] = dens(k + 2, hi);
  return CVA_OK;
}

int cva_cag_density_budget(int32_t chunk_index, int32_t hist_frames, int32_t blocks_per_frame,
                           int32_t k_f_max, double density, int32_t* k_f, int32_t* k_b) {
  if (!k_f || !k_b) return fail(CVA_EINVAL, "k_f or k_b is NULL");
  if (hist_frames < 0 || blocks_per_frame < 1 || k_f_max < 0 || !(density >= 0.0 && density <= 1.0))
    return fail(CVA_EINVAL, "bad budget arguments");
  const int64_t all = (int64_t)hist_frames * blocks_per_frame;
  if (chunk_index <= 1 || hist_frames == 0) {
    *k_f = hist_frames;
    *k_b = (int32_t)all;
    return CVA_OK;
  }
  const int kf = k_f_max < hist_frames ? k_f_max : hist_frames;
  int64_t kb = (int64_t)floor(density * (double)all + 0.5);
  const int64_t cand = (int64_t)kf * blocks_per_frame;
  if (kb > cand) kb = cand;
  *k_f = kf;
  *k_b = (int32_t)kb;
  return CVA_OK;
}

int cva_chunk_workspace_bytes(const cva_shape* shape, int32_t k_f, int32_t k_b, size_t* bytes) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!bytes) return fail(CVA_EINVAL, "bytes is NULL");
  const Dims d = make_dims(*shape);
  *bytes = chunk_ws_layout(d, k_f, k_b).total;
  return CVA_OK;
}

}  // extern "C"

// Every host check of the fused chunk call except those of the workspace;
// *ws_need gets the workspace bytes the call needs.
int cva::check_chunk_call(const void* q, const void* k, const void* v, const cva_kv_cache* cache,
                          const cva_rope_tables* tables, int32_t t0, int32_t k_f, int32_t k_b,
                          const void* out, size_t* ws_need) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (!q || !k || !v || !out) return fail(CVA_EINVAL, "NULL buffer");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
    return fail(CVA_EINVAL, "q, k, v and out must be 16-byte aligned");
  if (t0 < cache->t_begin) return fail(CVA_ERANGE, "t0 %d before the stream start %d", t0, cache->t_begin);
  const Dims d = make_dims(cache->shape);
  rc = check_tables(tables, d, t0);
  if (rc) return rc;
  const bool dense = k_f < 0;
  int t_lo, F;
  history(cache, t0, &t_lo, &F);
  if (!dense) {
    const int kfe = k_f < F ? k_f : F;
    if (F > 0 && k_f < 1) return fail(CVA_ERANGE, "k_f must be >= 1 when there is history");
    if (k_b < 0 || (int64_t)k_b > (int64_t)kfe * d.nb)
      return fail(CVA_ERANGE, "k_b %d outside [0, %d] (k_f_eff * blocks per frame)", k_b, kfe * d.nb);
    if (F > 256) return fail(CVA_ENOTSUP, "history frames %d > 256", F);
    if ((int64_t)kfe * d.nb > 1024) return fail(CVA_ENOTSUP, "candidate blocks %d > 1024", kfe * d.nb);
  }
  rc = check_attn_limits(d, F, dense || F == 0, dense ? 0 : k_b);
  if (rc) return rc;
  *ws_need = chunk_ws_layout(d, dense ? 0 : k_f, dense ? 0 : k_b).total;
  return CVA_OK;
}

// Steps 1-5 from q, k, v; topp > 0 selects blocks by the top-p budget with
// cap k_b.
static int chunk_attention_impl(const void* q, const void* k, const void* v, const cva_kv_cache* cache,
                                const cva_rope_tables* tables, int32_t t0, int32_t k_f, int32_t k_b,
                                float topp, void* workspace, size_t ws_bytes, void* out, float* lse,
                                cva_stream_t stream) {
  size_t need = 0;
  int rc = check_chunk_call(q, k, v, cache, tables, t0, k_f, k_b, out, &need);
  if (rc) return rc;
  if (!workspace) return fail(CVA_EINVAL, "workspace is NULL");
  if (!aligned(workspace, 256)) return fail(CVA_EINVAL, "workspace must be 256-byte aligned");
  if (ws_bytes < need) return fail(CVA_ENOMEM, "workspace %zu bytes < %zu needed", ws_bytes, need);
  const Dims d = make_dims(cache->shape);
  const bool dense = k_f < 0;
  const ChunkWs w = chunk_ws_layout(d, dense ? 0 : k_f, dense ? 0 : k_b);
  int t_lo, F;
  history(cache, t0, &t_lo, &F);

  char* ws = static_cast<char*>(workspace);
  uint16_t* q_rot = reinterpret_cast<uint16_t*>(ws + w.q_rot);
  float* qpool = reinterpret_cast<float*>(ws + w.qpool);
  int32_t* fidx = reinterpret_cast<int32_t*>(ws + w.frame_idx);
  int32_t* bidx = reinterpret_cast<int32_t*>(ws + w.block_idx);
  int32_t* bcnt = reinterpret_cast<int32_t*>(ws + w.block_cnt);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // steps 1-3: rotate Q (+ block pools) and K (+ append, block pools), copy V
  const RopePoolArgs a = chunk_rope_args(q, k, v, cache, tables, t0, q_rot, dense ? nullptr : qpool);
  cudaError_t e = stage_mark(0, s);
  if (e != cudaSuccess) return cuda_fail(e, "stage event");
  e = launch_rope_pool(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "chunk_attention rope/append launch");
  if ((e = stage_mark(1, s)) != cudaSuccess) return cuda_fail(e, "stage event");

  // step 4; each kernel from here on follows one of this call's kernels:
  // programmatic dependent launches, unless stage events sit between them
  const bool sparse = !dense && F > 0;
  const bool chain = !g_stage_on;
  const int32_t* qpair = nullptr;
  if (sparse) {
    rc = select_impl(qpool, cache, t0, k_f, k_b, fidx, bidx, bcnt, k_b, topp, s, chain);
    if (rc) return rc;
    rc = pair_impl(d, cache, t0, k_f, fidx, reinterpret_cast<int32_t*>(ws + w.qpair), &qpair, s, chain);
    if (rc) return rc;
  }
  if ((e = stage_mark(2, s)) != cudaSuccess) return cuda_fail(e, "stage event");
  // step 5 (with the frame means of the new cache frames)
  rc = attn_impl(q_rot, cache, t0, sparse ? bidx : nullptr, sparse ? bcnt : nullptr,
                 sparse ? k_b : 0, out, lse, ws + w.attn, attn_split_bytes(d), s, true, qpair, chain);
  if (rc) return rc;
  if ((e = stage_mark(3, s)) != cudaSuccess) return cuda_fail(e, "stage event");
  return CVA_OK;
}

extern "C" {

int cva_chunk_attention(const void* q, const void* k, const void* v, const cva_kv_cache* cache,
                        const cva_rope_tables* tables, int32_t t0, int32_t k_f, int32_t k_b,
                        void* workspace, size_t ws_bytes, void* out, float* lse,
                        cva_stream_t stream) {
  return chunk_attention_impl(q, k, v, cache, tables, t0, k_f, k_b, 0.f, workspace, ws_bytes, out, lse,
                              stream);
}

int cva_chunk_attention_topp(const void* q, const void* k, const void* v, const cva_kv_cache* cache,
                             const cva_rope_tables* tables, int32_t t0, int32_t k_f, int32_t k_cap,
                             float p, void* workspace, size_t ws_bytes, void* out, float* lse,
                             cva_stream_t stream) {
  if (!topp_ok(p)) return fail(CVA_ERANGE, "p must lie in (0, 1]");
  if (k_f < 1 || k_cap < 1) return fail(CVA_ERANGE, "k_f and k_cap must be >= 1");
  return chunk_attention_impl(q, k, v, cache, tables, t0, k_f, k_cap, p, workspace, ws_bytes, out, lse,
                              stream);
}

}  // extern "C"
