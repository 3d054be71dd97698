"""The whole per-chunk path over a frame cache (fp64).

Test infrastructure only (see :mod:`oracle`).

For every new chunk (Self-Forcing style chunk-by-chunk generation with a KV
cache and a rolling window, "Accelerating Video Generation Inference ...",
section 1) the path:

1. rotates Q and K with the global time index (:mod:`oracle.rope`);
2. appends the rotated K and V of the chunk's frames to the cache, evicting
   frames that fall out of a window of ``W`` frames (the window counts the
   current chunk's frames);
3. mean-pools Q per block and K per block and per frame;
4. picks frames, then blocks, per query block (:mod:`oracle.hsa`);
5. attends over the picked history blocks plus the whole current chunk
   (:mod:`oracle.attention`).

``store="bf16"`` rounds the rotated Q and K to bfloat16 (nearest, ties to
even) where the library stores them, so that every later step sees the
values the library keeps; ``store="f64"`` keeps the exact values.
"""
from __future__ import annotations

import math
from typing import Dict, Optional

import numpy as np

from . import rope as _rope
from . import hsa as _hsa
from .attention import attend


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 value (ties to even), exactly.

    bfloat16 keeps 8 significant bits; with ``x = m * 2**e`` and ``m`` in
    [0.5, 1), ``m * 2**8`` is rounded to an integer (numpy's ``rint`` rounds
    halves to even) and scaled back. Values below the smallest normal
    (2**-126) keep the same absolute quantum as at 2**-126.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    e = np.maximum(e, -125)                 # subnormal range: fixed quantum 2**-133
    return np.ldexp(np.rint(np.ldexp(x, 8 - e)), e - 8)


class FrameCache:
    """Rotated K and V per global frame index, with block and frame K pools."""

    def __init__(self, B: int, H: int, D: int, T_f: int, blk: int, window: int):
        self.B, self.H, self.D, self.T_f, self.blk, self.W = B, H, D, T_f, blk, window
        self.nb = -(-T_f // blk)
        self.frames: Dict[int, dict] = {}
        self.t_begin: Optional[int] = None

    def append(self, k_rot: np.ndarray, v: np.ndarray, t0: int, Fc: int) -> None:
        """Store frames ``t0 .. t0+Fc-1`` from ``[B, Lq, H, D]`` tensors, then evict
        every frame older than the newest ``W``."""
        T_f = self.T_f
        if self.t_begin is None:
            self.t_begin = t0
        for f in range(Fc):
            kf = np.transpose(k_rot[:, f * T_f:(f + 1) * T_f], (0, 2, 1, 3))  # [B,H,T_f,D]
            vf = np.transpose(v[:, f * T_f:(f + 1) * T_f], (0, 2, 1, 3))
            self.frames[t0 + f] = {
                "k": np.asarray(kf, dtype=np.float64),
                "v": np.asarray(vf, dtype=np.float64),
                "kb": _hsa.block_means(kf, self.blk),     # [B,H,nb,D]
                "kf": _hsa.frame_mean(kf),                # [B,H,D]
            }
        newest = t0 + Fc - 1
        for t in [t for t in self.frames if t <= newest - self.W]:
            del self.frames[t]

    def history(self, t0: int, Fc: int):
        """Global indices (ascending) of the history frames a chunk at ``t0`` sees:
        ``max(t_begin, t0 + Fc - W) .. t0 - 1``, where ``t_begin`` is the first
        frame the cache ever received (the stream's start offset)."""
        if not self.frames:
            return np.zeros(0, dtype=np.int64)
        t_begin = self.t_begin
        lo = max(t_begin, t0 + Fc - self.W)
        ts = list(range(lo, t0))
        missing = [t for t in ts if t not in self.frames]
        if missing:
            raise KeyError(f"history frames missing from cache: {missing[:4]}")
        return np.array(ts, dtype=np.int64)


def pool_queries(q_rot: np.ndarray, T_f: int, blk: int, Fc: int):
    """Block-pooled and frame-pooled queries of a chunk ``q_rot[B, Lq, H, D]``:
    ``[B, H, Fc*nb, D]`` and ``[B, H, Fc, D]``."""
    B, Lq, H, D = q_rot.shape
    qh = np.transpose(np.asarray(q_rot, dtype=np.float64), (0, 2, 1, 3)).reshape(B, H, Fc, T_f, D)
    qb = _hsa.block_means(qh, blk)                 # [B,H,Fc,nb,D]
    return qb.reshape(B, H, -1, D), _hsa.frame_mean(qh)


def select_chunk(qbar_blk: np.ndarray, cache: FrameCache, hist_t: np.ndarray,
                 k_f: int, k_b: int, topp: Optional[float] = None):
    """Two-level selection for every (b, h, query block).

    Returns ``frames [B,H,NQB,k_f_eff]``, ``blocks [B,H,NQB,k_b]`` (ids
    ``t*nb + j``, ascending) and the relative boundary gaps ``gap_f``,
    ``gap_b`` ``[B,H,NQB]`` (``inf`` where nothing was cut). With ``topp``
    the second level is :func:`oracle.hsa.block_select_topp` with cap
    ``k_b``: each row holds its chosen ids first, then ``-1``.
    """
    B, H, NQB, D = qbar_blk.shape
    nb = cache.nb
    F = hist_t.shape[0]
    k_f_eff = min(k_f, F)
    frames = np.zeros((B, H, NQB, k_f_eff), dtype=np.int64)
    blocks = np.full((B, H, NQB, k_b), -1 if topp is not None else 0, dtype=np.int64)
    gap_f = np.full((B, H, NQB), math.inf)
    gap_b = np.full((B, H, NQB), math.inf)
    if F:
        kf_all = np.stack([cache.frames[t]["kf"] for t in hist_t], axis=2)   # [B,H,F,D]
        kb_all = np.stack([cache.frames[t]["kb"] for t in hist_t], axis=2)   # [B,H,F,nb,D]
    for b in range(B):
        for h in range(H):
            for qb in range(NQB):
                if F == 0:
                    continue
                ft, gf = _hsa.frame_select(qbar_blk[b, h, qb], kf_all[b, h], hist_t, k_f)
                pos = np.searchsorted(hist_t, ft)
                if topp is None:
                    ids, gb = _hsa.block_select(qbar_blk[b, h, qb], kb_all[b, h][pos], ft, nb, k_b)
                else:
                    ids, gb = _hsa.block_select_topp(qbar_blk[b, h, qb], kb_all[b, h][pos], ft, nb,
                                                     cache.T_f, cache.blk, topp, k_b)
                frames[b, h, qb] = ft
                blocks[b, h, qb, :len(ids)] = ids
                gap_f[b, h, qb] = gf
                gap_b[b, h, qb] = gb
    return frames, blocks, gap_f, gap_b


def keys_of_query_block(cache: FrameCache, b: int, h: int, t0: int, Fc: int,
                        block_ids: Optional[np.ndarray]):
    """K and V rows a query block attends to: the valid tokens of its picked
    history blocks (all history blocks when ``block_ids`` is None) followed by
    every token of the current chunk's frames. Negative ids (list padding)
    are skipped."""
    nb, blk, T_f = cache.nb, cache.blk, cache.T_f
    ks, vs = [], []
    if block_ids is None:
        hist = cache.history(t0, Fc)
        block_ids = (hist[:, None] * nb + np.arange(nb)[None, :]).reshape(-1)
    for g in np.asarray(block_ids):
        if g < 0:
            continue
        t, j = divmod(int(g), nb)
        fr = cache.frames[t]
        lo, hi = j * blk, min((j + 1) * blk, T_f)
        ks.append(fr["k"][b, h, lo:hi])
        vs.append(fr["v"][b, h, lo:hi])
    for t in range(t0, t0 + Fc):
        ks.append(cache.frames[t]["k"][b, h])
        vs.append(cache.frames[t]["v"][b, h])
    return np.concatenate(ks, axis=0), np.concatenate(vs, axis=0)


def attend_chunk(q_rot: np.ndarray, cache: FrameCache, t0: int, Fc: int,
                 blocks: Optional[np.ndarray], rows=None):
    """Attention of a chunk's queries ``q_rot[B, Lq, H, D]``.

    ``blocks[B, H, NQB, k_b]`` are the picked history block ids per query
    block (None: every history block). ``rows`` optionally restricts the
    queries to a list of token indices. Returns ``o[B, Lq, H, D]`` and
    ``lse[B, H, Lq]`` (NaN where not computed).
    """
    B, Lq, H, D = q_rot.shape
    T_f, blk, nb = cache.T_f, cache.blk, cache.nb
    scale = 1.0 / math.sqrt(D)
    o = np.full((B, Lq, H, D), np.nan)
    lse = np.full((B, H, Lq), np.nan)
    rows = np.arange(Lq) if rows is None else np.asarray(rows)
    qb_of_row = (rows // T_f) * nb + (rows % T_f) // blk
    for b in range(B):
        for h in range(H):
            for qb in np.unique(qb_of_row):
                r = rows[qb_of_row == qb]
                ids = None if blocks is None else blocks[b, h, qb]
                k, v = keys_of_query_block(cache, b, h, t0, Fc, ids)
                oo, ll = attend(np.asarray(q_rot[b, r, h], dtype=np.float64), k, v, scale)
                o[b, r, h] = oo
                lse[b, h, r] = ll
    return o, lse


def rotate_chunk(q: np.ndarray, k: np.ndarray, Fh: int, Fw: int, Fc: int, t0: int,
                 store: str = "bf16"):
    """Causal-RoPE of a chunk's Q and K, rounded to bfloat16 when ``store='bf16'``."""
    q_rot = _rope.rope_chunk(q, Fh, Fw, Fc, t0)
    k_rot = _rope.rope_chunk(k, Fh, Fw, Fc, t0)
    if store == "bf16":
        q_rot, k_rot = round_bf16(q_rot), round_bf16(k_rot)
    return q_rot, k_rot


def run_chunk(cache: FrameCache, q: np.ndarray, k: np.ndarray, v: np.ndarray, *,
              Fh: int, Fw: int, Fc: int, t0: int, k_f: int, k_b: int,
              dense: bool, store: str = "bf16", rows=None, attend_too: bool = True,
              topp: Optional[float] = None):
    """One chunk through the whole path; returns every intermediate.

    ``q, k, v`` are the raw ``[B, Lq, H, D]`` inputs (fp64 values). The cache
    is updated in place. ``topp`` switches the second selection level to the
    top-p budget with cap ``k_b``.
    """
    q_rot, k_rot = rotate_chunk(q, k, Fh, Fw, Fc, t0, store)
    cache.append(k_rot, np.asarray(v, dtype=np.float64), t0, Fc)
    hist = cache.history(t0, Fc)
    qbar_blk, qbar_frm = pool_queries(q_rot, cache.T_f, cache.blk, Fc)
    out = {"q_rot": q_rot, "k_rot": k_rot, "qbar_blk": qbar_blk, "qbar_frm": qbar_frm,
           "hist": hist}
    if dense:
        out.update(frames=None, blocks=None, gap_f=None, gap_b=None)
        blocks = None
    else:
        frames, blocks, gf, gb = select_chunk(qbar_blk, cache, hist, k_f, k_b, topp)
        out.update(frames=frames, blocks=blocks, gap_f=gf, gap_b=gb)
    if attend_too:
        o, lse = attend_chunk(q_rot, cache, t0, Fc, blocks, rows)
        out.update(o=o, lse=lse)
    return out
