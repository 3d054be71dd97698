"""ctypes binding of ``libcva.so`` (the C ABI declared in ``include/cva.h``).

Argument marshalling only: every step of the path runs in the library's
CUDA kernels. Tensors are torch tensors on the device (torch provides the
memory and the stream); shapes and layouts are those of the header. There
is no CPU fallback: importing this module without the built library raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcva.so")

c_int32 = ctypes.c_int32
c_int64 = ctypes.c_int64
c_void_p = ctypes.c_void_p
c_size_t = ctypes.c_size_t

# status codes (cva.h)
CVA_OK, CVA_EINVAL, CVA_ENOTSUP, CVA_ERANGE, CVA_ENOMEM, CVA_ELAUNCH, CVA_EDEVICE = 0, -1, -2, -3, -4, -5, -6
DEV_OK, DEV_TIMEOUT, DEV_BAD_INDEX, DEV_BAD_COUNT = 0, 1, 2, 3


class CvaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libcva error {code}: {msg}")
        self.code = code


class Shape(ctypes.Structure):
    _fields_ = [("batch", c_int32), ("heads", c_int32), ("head_dim", c_int32),
                ("frame_h", c_int32), ("frame_w", c_int32), ("chunk_frames", c_int32),
                ("block", c_int32)]


class RopeCfg(ctypes.Structure):
    _fields_ = [("head_dim", c_int32), ("max_t", c_int32), ("frame_h", c_int32),
                ("frame_w", c_int32), ("theta", ctypes.c_double)]


class RopeTables(ctypes.Structure):
    _fields_ = [("cos_t", c_void_p), ("sin_t", c_void_p), ("cos_h", c_void_p),
                ("sin_h", c_void_p), ("cos_w", c_void_p), ("sin_w", c_void_p),
                ("max_t", c_int32), ("frame_h", c_int32), ("frame_w", c_int32),
                ("head_dim", c_int32), ("cs_tok", c_void_p)]


class KVCache(ctypes.Structure):
    _fields_ = [("k", c_void_p), ("v", c_void_p), ("kpool_blk", c_void_p),
                ("kpool_frm", c_void_p), ("window", c_int32), ("t_begin", c_int32),
                ("shape", Shape)]


class CagCfg(ctypes.Structure):
    _fields_ = [("dense", c_int32), ("k_f_max", c_int32), ("d_base_num", c_int64),
                ("d_base_den", c_int64), ("d_slope_num", c_int64), ("d_slope_den", c_int64),
                ("pivot", c_int32), ("k_b_fixed", c_int32)]


P = ctypes.POINTER
_SIGS = {
    "cva_version": (c_int32, []),
    "cva_last_error": (ctypes.c_char_p, []),
    "cva_device_status": (c_int32, [P(c_int32), c_int32]),
    "cva_rope_axis_pairs": (c_int32, [c_int32, P(c_int32), P(c_int32), P(c_int32)]),
    "cva_rope3d_precompute": (c_int32, [P(RopeCfg)] + [c_void_p] * 6),
    "cva_rope3d_precompute_tokens": (c_int32, [P(RopeCfg), c_void_p]),
    "cva_rope3d_apply": (c_int32, [c_void_p, c_void_p, P(RopeTables), P(Shape), c_int32, c_int32, c_void_p]),
    "cva_kv_append": (c_int32, [c_void_p, c_void_p, P(KVCache), P(RopeTables), c_int32, c_void_p]),
    "cva_rotate_append_pool": (c_int32, [c_void_p, c_void_p, c_void_p, P(KVCache), P(RopeTables), c_int32,
                                         c_void_p, c_void_p, c_void_p]),
    "cva_kv_frame_means": (c_int32, [P(KVCache), c_int32, c_void_p]),
    "cva_history_frames": (c_int32, [P(KVCache), c_int32, P(c_int32), P(c_int32)]),
    "cva_qkv_rope_append": (c_int32, [c_void_p, c_void_p, c_int32, P(KVCache), P(RopeTables), c_int32,
                                      c_void_p, c_void_p, c_void_p]),
    "cva_cag_noise_densities": (c_int32, [c_int32, c_int32, c_int32, c_int32, ctypes.c_double,
                                          ctypes.c_double, c_void_p]),
    "cva_cag_density_budget": (c_int32, [c_int32, c_int32, c_int32, c_int32, ctypes.c_double, P(c_int32),
                                         P(c_int32)]),
    "cva_chunk_attention_qkv": (c_int32, [c_void_p, c_void_p, c_int32, P(KVCache), P(RopeTables), c_int32,
                                          c_int32, c_int32, c_void_p, ctypes.c_size_t, c_void_p, c_void_p,
                                          c_void_p]),
    "cva_hsa_compress": (c_int32, [c_void_p, P(Shape), c_void_p, c_void_p, c_void_p]),
    "cva_hsa_select": (c_int32, [c_void_p, P(KVCache), c_int32, c_int32, c_int32, c_void_p,
                                 c_void_p, c_void_p, c_void_p]),
    "cva_hsa_select_topp": (c_int32, [c_void_p, P(KVCache), c_int32, c_int32, c_int32, ctypes.c_float,
                                      c_void_p, c_void_p, c_void_p, c_void_p]),
    "cva_attn_workspace_bytes": (c_int32, [P(Shape), c_int32, P(c_size_t)]),
    "cva_blocksparse_attn_fwd": (c_int32, [c_void_p, P(KVCache), c_int32, c_void_p, c_void_p,
                                           c_int32, c_void_p, c_void_p, c_void_p, c_size_t,
                                           c_void_p]),
    "cva_chunk_workspace_bytes": (c_int32, [P(Shape), c_int32, c_int32, P(c_size_t)]),
    "cva_chunk_attention": (c_int32, [c_void_p, c_void_p, c_void_p, P(KVCache), P(RopeTables),
                                      c_int32, c_int32, c_int32, c_void_p, c_size_t, c_void_p,
                                      c_void_p, c_void_p]),
    "cva_chunk_attention_topp": (c_int32, [c_void_p, c_void_p, c_void_p, P(KVCache), P(RopeTables),
                                           c_int32, c_int32, c_int32, ctypes.c_float, c_void_p, c_size_t,
                                           c_void_p, c_void_p, c_void_p]),
    "cva_chunk_attention_noalloc": (c_int32, [c_void_p, c_void_p, c_void_p, P(KVCache), P(RopeTables),
                                              c_int32, c_int32, c_int32, c_void_p, c_void_p, c_void_p]),
    "cva_copy_rows_2d": (c_int32, [c_void_p, c_void_p] + [ctypes.c_int64] * 7 + [c_void_p]),
    "cva_set_stage_events": (c_int32, [P(c_void_p), c_int32]),
    "cva_diag_wait_timeout": (c_int32, [c_int32, c_void_p, c_void_p]),
    "cva_diag_mma_cycles": (c_int32, [c_int32, c_int32, c_int32, c_void_p, c_int32, c_void_p]),
    "cva_kv_cache_bytes": (c_int32, [P(Shape), c_int32, P(c_size_t)]),
    "cva_kv_cache_init": (c_int32, [P(KVCache), c_void_p, c_size_t, P(Shape), c_int32, c_int32]),
    "cva_cag_budget": (c_int32, [P(CagCfg), c_int32, c_int32, c_int32, P(c_int32), P(c_int32)]),
}


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"libcva.so not built ({_LIB_PATH}); run `python -m autoregressive_video_dit_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()
EXPORTED = tuple(_SIGS)


def last_error() -> str:
    return lib.cva_last_error().decode()


def check(rc: int) -> None:
    if rc != CVA_OK:
        raise CvaError(rc, last_error())


# --- helpers ----------------------------------------------------------------

def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _stream(stream) -> int:
    import torch
    if stream is None:
        return int(torch.cuda.current_stream().cuda_stream)
    return int(stream.cuda_stream if hasattr(stream, "cuda_stream") else stream)


def make_shape(B, H, D, Fh, Fw, Fc, blk) -> Shape:
    return Shape(B, H, D, Fh, Fw, Fc, blk)


def dims(shape: Shape) -> dict:
    T_f = shape.frame_h * shape.frame_w
    nb = -(-T_f // shape.block)
    return {"T_f": T_f, "nb": nb, "T_pad": nb * shape.block, "Lq": shape.chunk_frames * T_f,
            "NQB": shape.chunk_frames * nb}


# --- host-only entry points ---------------------------------------------------

def rope_axis_pairs(head_dim: int) -> Tuple[int, int, int]:
    a, b, c = c_int32(), c_int32(), c_int32()
    check(lib.cva_rope_axis_pairs(head_dim, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)))
    return a.value, b.value, c.value


def rope3d_precompute(head_dim: int, max_t: int, frame_h: int, frame_w: int,
                      theta: float = 10000.0) -> dict:
    """Host cos/sin tables (float32 numpy arrays), one [positions, pairs] pair per axis."""
    pt, ph, pw = rope_axis_pairs(head_dim)
    out = {"cos_t": np.zeros((max_t, pt), np.float32), "sin_t": np.zeros((max_t, pt), np.float32),
           "cos_h": np.zeros((frame_h, ph), np.float32), "sin_h": np.zeros((frame_h, ph), np.float32),
           "cos_w": np.zeros((frame_w, pw), np.float32), "sin_w": np.zeros((frame_w, pw), np.float32)}
    cfg = RopeCfg(head_dim, max_t, frame_h, frame_w, theta)
    check(lib.cva_rope3d_precompute(ctypes.byref(cfg), *[out[k].ctypes.data for k in
                                                          ("cos_t", "sin_t", "cos_h", "sin_h",
                                                           "cos_w", "sin_w")]))
    out["cs_tok"] = np.zeros((frame_h, frame_w, head_dim // 2, 2), np.float32)
    check(lib.cva_rope3d_precompute_tokens(ctypes.byref(cfg), out["cs_tok"].ctypes.data))
    return out


def cag_budget(chunk_index: int, hist_frames: int, blocks_per_frame: int, *, dense: bool,
               k_f_max: int = 0, d_base=(0, 1), d_slope=(0, 1), pivot: int = 0,
               k_b_fixed: Optional[int] = None) -> Tuple[int, int]:
    """(k_f, k_b) of one chunk; densities are (numerator, denominator) pairs."""
    cfg = CagCfg(int(dense), k_f_max, d_base[0], d_base[1], d_slope[0], d_slope[1], pivot,
                 -1 if k_b_fixed is None else int(k_b_fixed))
    kf, kb = c_int32(), c_int32()
    check(lib.cva_cag_budget(ctypes.byref(cfg), chunk_index, hist_frames, blocks_per_frame,
                             ctypes.byref(kf), ctypes.byref(kb)))
    return kf.value, kb.value


def kv_cache_bytes(shape: Shape, window: int) -> int:
    n = c_size_t()
    check(lib.cva_kv_cache_bytes(ctypes.byref(shape), window, ctypes.byref(n)))
    return n.value


def chunk_workspace_bytes(shape: Shape, k_f: int, k_b: int) -> int:
    n = c_size_t()
    check(lib.cva_chunk_workspace_bytes(ctypes.byref(shape), k_f, k_b, ctypes.byref(n)))
    return n.value


def attn_workspace_bytes(shape: Shape, k_b_max: int) -> int:
    n = c_size_t()
    check(lib.cva_attn_workspace_bytes(ctypes.byref(shape), k_b_max, ctypes.byref(n)))
    return n.value


def set_stage_events(events) -> None:
    """Record 4 torch.cuda.Event objects around the stages of chunk_attention (None: stop)."""
    if events is None:
        check(lib.cva_set_stage_events(None, 0))
        return
    arr = (c_void_p * 4)(*[int(e.cuda_event) for e in events])
    check(lib.cva_set_stage_events(arr, len(events)))


def diag_mma_cycles(m: int, n: int, iters: int, cycles, stream=None) -> None:
    """Diagnostic: clock64 span of iters x 4 back-to-back m x n x 16 MMAs per
    CTA, one CTA per element of the uint64 (int64) device tensor `cycles`."""
    check(lib.cva_diag_mma_cycles(m, n, iters, _ptr(cycles), cycles.numel(), _stream(stream)))


def diag_wait_timeout(limit_us: int, result, stream=None) -> None:
    """Diagnostic: a bounded wait on an mbarrier nothing arrives at (see cva.h);
    result is an int32 device tensor of 2 elements."""
    check(lib.cva_diag_wait_timeout(limit_us, _ptr(result), _stream(stream)))


def device_status(clear: bool = True) -> int:
    code = c_int32()
    check(lib.cva_device_status(ctypes.byref(code), int(clear)))
    return code.value


# --- device objects ------------------------------------------------------------

class DeviceRopeTables:
    """The rotary tables copied to the device once (precomputed contiguous tables)."""

    def __init__(self, head_dim: int, max_t: int, frame_h: int, frame_w: int,
                 theta: float = 10000.0, device="cuda"):
        import torch
        host = rope3d_precompute(head_dim, max_t, frame_h, frame_w, theta)
        self.tensors = {k: torch.from_numpy(v).to(device) for k, v in host.items()}
        t = self.tensors
        self.struct = RopeTables(_ptr(t["cos_t"]), _ptr(t["sin_t"]), _ptr(t["cos_h"]),
                                 _ptr(t["sin_h"]), _ptr(t["cos_w"]), _ptr(t["sin_w"]),
                                 max_t, frame_h, frame_w, head_dim, _ptr(t["cs_tok"]))


class DeviceKVCache:
    """One layer's frame cache: torch owns the arena, the library lays it out."""

    def __init__(self, shape: Shape, window: int, t_begin: int = 0, device="cuda", arena=None):
        import torch
        nbytes = kv_cache_bytes(shape, window)
        if arena is None:
            arena = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        self.arena = arena
        self.struct = KVCache()
        check(lib.cva_kv_cache_init(ctypes.byref(self.struct), _ptr(arena), nbytes,
                                    ctypes.byref(shape), window, t_begin))
        self.shape = shape
        self.window = window
        self.t_begin = t_begin
        dd = dims(shape)
        B, H, D = shape.batch, shape.heads, shape.head_dim
        base = _ptr(arena)

        def view(ptr, n, dtype, shp):
            off = ptr - base
            esz = torch.tensor([], dtype=dtype).element_size()
            return arena[off:off + n * esz].view(dtype).view(shp)

        self.k = view(self.struct.k, B * H * window * dd["T_pad"] * D, torch.bfloat16,
                      (B, H, window, dd["T_pad"], D))
        self.v = view(self.struct.v, B * H * window * dd["T_pad"] * D, torch.bfloat16,
                      (B, H, window, dd["T_pad"], D))
        self.kpool_blk = view(self.struct.kpool_blk, B * H * window * dd["nb"] * D, torch.float32,
                              (B, H, window, dd["nb"], D))
        self.kpool_frm = view(self.struct.kpool_frm, B * H * window * D, torch.float32,
                              (B, H, window, D))

    def history_frames(self, t0: int) -> Tuple[int, int]:
        lo, n = c_int32(), c_int32()
        check(lib.cva_history_frames(ctypes.byref(self.struct), t0, ctypes.byref(lo), ctypes.byref(n)))
        return lo.value, n.value


# --- device entry points (same names as the C ABI) ---------------------------------

def rope3d_apply(x, y, tables: DeviceRopeTables, shape: Shape, t0: int, out_layout: int = 0,
                 stream=None) -> None:
    check(lib.cva_rope3d_apply(_ptr(x), _ptr(y), ctypes.byref(tables.struct), ctypes.byref(shape),
                               t0, out_layout, _stream(stream)))


def kv_append(k, v, cache: DeviceKVCache, tables: Optional[DeviceRopeTables], t0: int,
              stream=None) -> None:
    check(lib.cva_kv_append(_ptr(k), _ptr(v), ctypes.byref(cache.struct),
                            None if tables is None else ctypes.byref(tables.struct), t0,
                            _stream(stream)))


def rotate_append_pool(q, k, v, cache: DeviceKVCache, tables: DeviceRopeTables, t0: int, q_rot,
                       qpool_blk=None, stream=None) -> None:
    """Steps 1-3 of chunk_attention in its single launch (see cva.h); the frame
    means of the new frames come from kv_frame_means or chunk_attention."""
    check(lib.cva_rotate_append_pool(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(cache.struct),
                                     ctypes.byref(tables.struct), t0, _ptr(q_rot), _ptr(qpool_blk),
                                     _stream(stream)))


def kv_frame_means(cache: DeviceKVCache, t0: int, stream=None) -> None:
    check(lib.cva_kv_frame_means(ctypes.byref(cache.struct), t0, _stream(stream)))


def qkv_rope_append(x, w_qkv, cache: DeviceKVCache, tables: DeviceRopeTables, t0: int, q_rot,
                    qpool_blk=None, stream=None) -> None:
    """x: bf16 [B, Lq, C]; w_qkv: bf16 [3*H*D, C]; q_rot: bf16 [B][H][Fc*T_pad][D] (output)."""
    check(lib.cva_qkv_rope_append(_ptr(x), _ptr(w_qkv), int(x.shape[-1]), ctypes.byref(cache.struct),
                                  ctypes.byref(tables.struct), t0, _ptr(q_rot), _ptr(qpool_blk),
                                  _stream(stream)))


def chunk_attention_qkv(x, w_qkv, cache: DeviceKVCache, tables: DeviceRopeTables, t0: int, k_f: int,
                        k_b: int, workspace, out, lse=None, stream=None) -> None:
    """chunk_attention starting from the hidden states x [B, Lq, C] and the
    fused projection weight w_qkv [3*H*D, C]."""
    ws_bytes = workspace.numel() * workspace.element_size()
    check(lib.cva_chunk_attention_qkv(_ptr(x), _ptr(w_qkv), int(x.shape[-1]), ctypes.byref(cache.struct),
                                      ctypes.byref(tables.struct), t0, k_f, k_b, _ptr(workspace), ws_bytes,
                                      _ptr(out), _ptr(lse), _stream(stream)))


def cag_noise_densities(n_chunks: int, Fc: int, window: int, blocks_per_frame: int, s_base: float,
                        s_target: float) -> dict:
    """{chunk: density} for chunks 2..n_chunks (see cva.h)."""
    buf = (ctypes.c_double * (n_chunks - 1))()
    check(lib.cva_cag_noise_densities(n_chunks, Fc, window, blocks_per_frame, s_base, s_target, buf))
    return {i + 2: buf[i] for i in range(n_chunks - 1)}


def cag_density_budget(chunk: int, hist_frames: int, blocks_per_frame: int, k_f_max: int,
                       density: float) -> Tuple[int, int]:
    kf, kb = c_int32(), c_int32()
    check(lib.cva_cag_density_budget(chunk, hist_frames, blocks_per_frame, k_f_max, density,
                                     ctypes.byref(kf), ctypes.byref(kb)))
    return kf.value, kb.value


def hsa_compress(q_rot, shape: Shape, qpool_blk, qpool_frm=None, stream=None) -> None:
    check(lib.cva_hsa_compress(_ptr(q_rot), ctypes.byref(shape), _ptr(qpool_blk), _ptr(qpool_frm),
                               _stream(stream)))


def hsa_select(qpool_blk, cache: DeviceKVCache, t0: int, k_f: int, k_b: int, frame_idx,
               block_idx, block_cnt, stream=None) -> None:
    check(lib.cva_hsa_select(_ptr(qpool_blk), ctypes.byref(cache.struct), t0, k_f, k_b,
                             _ptr(frame_idx), _ptr(block_idx), _ptr(block_cnt), _stream(stream)))


def hsa_select_topp(qpool_blk, cache: DeviceKVCache, t0: int, k_f: int, k_cap: int, p: float, frame_idx,
                    block_idx, block_cnt, stream=None) -> None:
    """Selection with the top-p block budget (cap k_cap, threshold p)."""
    check(lib.cva_hsa_select_topp(_ptr(qpool_blk), ctypes.byref(cache.struct), t0, k_f, k_cap, p,
                                  _ptr(frame_idx), _ptr(block_idx), _ptr(block_cnt), _stream(stream)))


def blocksparse_attn_fwd(q_rot, cache: DeviceKVCache, t0: int, block_idx, block_cnt, k_b_max: int,
                         out, lse=None, workspace=None, stream=None) -> None:
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    check(lib.cva_blocksparse_attn_fwd(_ptr(q_rot), ctypes.byref(cache.struct), t0,
                                       _ptr(block_idx), _ptr(block_cnt), k_b_max, _ptr(out),
                                       _ptr(lse), _ptr(workspace), ws_bytes, _stream(stream)))


def chunk_attention(q, k, v, cache: DeviceKVCache, tables: DeviceRopeTables, t0: int, k_f: int,
                    k_b: int, workspace, out, lse=None, stream=None) -> None:
    ws_bytes = workspace.numel() * workspace.element_size()
    check(lib.cva_chunk_attention(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(cache.struct),
                                  ctypes.byref(tables.struct), t0, k_f, k_b, _ptr(workspace),
                                  ws_bytes, _ptr(out), _ptr(lse), _stream(stream)))


def chunk_attention_topp(q, k, v, cache: DeviceKVCache, tables: DeviceRopeTables, t0: int, k_f: int,
                         k_cap: int, p: float, workspace, out, lse=None, stream=None) -> None:
    """chunk_attention with the top-p block budget of hsa_select_topp."""
    ws_bytes = workspace.numel() * workspace.element_size()
    check(lib.cva_chunk_attention_topp(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(cache.struct),
                                       ctypes.byref(tables.struct), t0, k_f, k_cap, p, _ptr(workspace),
                                       ws_bytes, _ptr(out), _ptr(lse), _stream(stream)))


def copy_rows_2d(src, dst, n0: int, n1: int, inner_bytes: int, src_strides, dst_strides, stream=None) -> None:
    """Batched row copies over an n0 x n1 index space (byte strides; see cva.h)."""
    check(lib.cva_copy_rows_2d(_ptr(src), _ptr(dst), n0, n1, inner_bytes, src_strides[0], src_strides[1],
                               dst_strides[0], dst_strides[1], _stream(stream)))


def chunk_attention_noalloc(q, k, v, cache: DeviceKVCache, tables: DeviceRopeTables, t0: int, k_f: int,
                            k_b: int, out, lse=None, stream=None) -> None:
    """chunk_attention with the library's fixed scratch instead of a workspace
    (for callers that cannot allocate device memory; see cva.h)."""
    check(lib.cva_chunk_attention_noalloc(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(cache.struct),
                                          ctypes.byref(tables.struct), t0, k_f, k_b, _ptr(out),
                                          _ptr(lse), _stream(stream)))
