"""Helpers shared by the GPU parity tests.

They move seeded inputs to the device and back, and drive the fp64 oracle
over the same chunks. No expected value here comes from the CUDA path.
"""
from __future__ import annotations

import math

import numpy as np

from cva_workload import WORKLOADS, Workload, chunk_inputs, bf16_bits_to_f32, key_centres
from oracle import hsa as o_hsa
from oracle import path as o_path


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(bits).astype(np.float64)


def f64_to_bits(x: np.ndarray) -> np.ndarray:
    """Exact bits of values that are already bfloat16-representable."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value is not a bfloat16"
    return (u >> 16).astype(np.uint16)


def to_dev(bits: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def from_dev(t) -> np.ndarray:
    import torch
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def shape_of(wl: Workload):
    from autoregressive_video_dit_b200 import ops
    return ops.make_shape(wl.B, wl.H, wl.D, wl.Fh, wl.Fw, wl.Fc, wl.blk)


def hist_count(wl: Workload, chunk: int, t_begin: int = 0) -> int:
    t0 = wl.t0_of(chunk) + t_begin
    lo = max(t_begin, t0 + wl.Fc - wl.window)
    return max(0, t0 - lo)


def oracle_budget(wl: Workload, chunk: int, t_begin: int = 0):
    return o_hsa.budget(chunk, hist_count(wl, chunk, t_begin), wl.nb, dense=wl.dense,
                        k_f_max=wl.k_f_max, d_base=wl.d_base, d_slope=wl.d_slope,
                        d_pivot=wl.d_pivot, k_b_fixed=wl.k_b_fixed)


def lib_budget(wl: Workload, chunk: int, t_begin: int = 0):
    from autoregressive_video_dit_b200 import ops
    return ops.cag_budget(chunk, hist_count(wl, chunk, t_begin), wl.nb, dense=wl.dense,
                          k_f_max=wl.k_f_max,
                          d_base=(wl.d_base.numerator, wl.d_base.denominator),
                          d_slope=(wl.d_slope.numerator, wl.d_slope.denominator),
                          pivot=wl.d_pivot, k_b_fixed=wl.k_b_fixed)


def inputs(wl: Workload, chunk: int, layer: int = 0, heads=None, centres=None):
    x = chunk_inputs(wl, chunk, layer, centres=centres)
    if heads is not None:
        for n in ("q", "k", "v"):
            x[n] = np.ascontiguousarray(x[n][:, :, heads])
    return x


def oracle_history(wl: Workload, chunk: int, layer: int = 0, heads=None, t_begin: int = 0,
                   store="bf16"):
    """Oracle frame cache after appending chunks 1..chunk-1 (only those the
    window keeps are drawn)."""
    H = wl.H if heads is None else len(heads)
    cache = o_path.FrameCache(wl.B, H, wl.D, wl.T_f, wl.blk, wl.window)
    centres = key_centres(wl, layer) if wl.keys == "clustered" else None
    cache.t_begin = t_begin
    t0_cur = wl.t0_of(chunk) + t_begin
    lo = max(t_begin, t0_cur + wl.Fc - wl.window)
    first = (lo - t_begin) // wl.Fc + 1
    for c in range(first, chunk):
        x = inputs(wl, c, layer, heads, centres)
        q, k, v = (bits_to_f64(x[n]) for n in ("q", "k", "v"))
        t0 = wl.t0_of(c) + t_begin
        _, k_rot = o_path.rotate_chunk(q, k, wl.Fh, wl.Fw, wl.Fc, t0, store)
        cache.append(k_rot, v, t0, wl.Fc)
    return cache


def sample_rows(wl: Workload, per_block: int, rng, blocks=None):
    """A few query rows from each (or the given) query block, including the
    first and last valid row of every sampled block."""
    rows = []
    qbs = range(wl.NQB) if blocks is None else blocks
    for qb in qbs:
        f, j = divmod(qb, wl.nb)
        lo = f * wl.T_f + j * wl.blk
        hi = f * wl.T_f + min((j + 1) * wl.blk, wl.T_f)
        pick = {lo, hi - 1}
        pick.update(int(r) for r in rng.integers(lo, hi, per_block))
        rows.extend(sorted(pick))
    return np.array(sorted(set(rows)))


def attn_errors(got: np.ndarray, want: np.ndarray):
    d = np.abs(got - want)
    rel_l2 = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))
    return float(d.max()), float(d.mean()), rel_l2


def valid_topk(scores: np.ndarray, chosen, k: int, tol: float) -> bool:
    """``chosen`` (positions into ``scores``) is a top-``k`` of ``scores`` up to
    near-ties: k distinct positions, every chosen score at least the k-th
    largest score minus ``delta`` and every other score at most the (k+1)-th
    plus ``delta``, with ``delta = tol * max(|s_k|, |s_k+1|)``. A set that is
    valid this way differs from the exact top-k only by swapping candidates
    whose scores lie within ``delta`` of the cut."""
    chosen = np.asarray(chosen, dtype=np.int64)
    n = scores.shape[0]
    if chosen.shape[0] != k or np.unique(chosen).shape[0] != k:
        return False
    if k == 0 or k == n:
        return True
    if chosen.min() < 0 or chosen.max() >= n:
        return False
    srt = np.sort(scores)[::-1]
    hi, lo = srt[k - 1], srt[k]
    delta = tol * max(abs(hi), abs(lo), 1e-30)
    inside = np.zeros(n, dtype=bool)
    inside[chosen] = True
    return bool(scores[inside].min() >= hi - delta and scores[~inside].max() <= lo + delta)


def check_selection(run, gpu_frames, gpu_blocks, gpu_cnt, tol=1e-5):
    """Compare the GPU's per-(b, h, query block) frame and block lists with the
    oracle's.

    A unit whose lists equal the oracle's is fine. A unit that differs is
    accepted only if the GPU's lists are still a valid two-level top-k under the
    oracle's own fp64 pooled scores (:func:`valid_topk`): its frames a valid
    top-k_f of the history frames, its blocks a valid top-k_b of the blocks of
    *its* frames, both ascending. Returns ``(n_units, n_bad, n_near, blocks)``:
    ``n_bad`` units that differ and are not valid, ``n_near`` units that differ
    validly, and the oracle's block lists with each such unit's list replaced by
    the GPU's (the key sets the GPU's attention must have used)."""
    o_blocks = run["blocks"]
    B, H, NQB, kb = o_blocks.shape
    cache, qbar = run["cache"], run["qbar_blk"]
    hist = np.asarray(run["hist_t"] if "hist_t" in run else run["hist"])
    nb = cache.nb
    F = hist.shape[0]
    kfe = run["frames"].shape[-1]
    blocks = o_blocks.copy()
    bad = near = 0
    for b in range(B):
        for h in range(H):
            kf_all = np.stack([cache.frames[t]["kf"][b, h] for t in hist]) if F else None
            for qb in range(NQB):
                gb = np.asarray(gpu_blocks[b, h, qb, :kb], dtype=np.int64)
                gf = np.asarray(gpu_frames[b, h, qb, :kfe], dtype=np.int64)
                if (gpu_cnt[b, h, qb] == kb and np.array_equal(gb, o_blocks[b, h, qb])
                        and np.array_equal(gf, run["frames"][b, h, qb])):
                    continue
                ok = gpu_cnt[b, h, qb] == kb and F > 0
                ok = ok and bool(np.all(np.diff(gf) > 0)) and bool(np.all(np.diff(gb) > 0))
                ok = ok and bool(np.all(np.isin(gf, hist)))
                if ok:
                    q = qbar[b, h, qb]
                    fpos = np.searchsorted(hist, gf)
                    ok = valid_topk(kf_all @ q, fpos, kfe, tol)
                if ok:
                    kb_sel = np.stack([cache.frames[int(t)]["kb"][b, h] for t in gf])   # [kfe, nb, D]
                    cand_ids = (gf[:, None] * nb + np.arange(nb)[None, :]).reshape(-1)
                    cand_s = kb_sel.reshape(-1, kb_sel.shape[-1]) @ q
                    ok = bool(np.all(np.isin(gb, cand_ids)))
                    ok = ok and valid_topk(cand_s, np.searchsorted(cand_ids, gb), kb, tol)
                if ok:
                    near += 1
                    blocks[b, h, qb] = gb
                else:
                    bad += 1
    return B * H * NQB, bad, near, blocks


def ws_lists(wl, ws, k_f, k_b, kfe):
    """Frame lists, block lists and counts the fused call wrote into its workspace
    (layout of cva_chunk_workspace_bytes: q_rot, pooled q, frames, blocks, counts)."""
    d = wl
    bhq = d.B * d.H * d.NQB
    r256 = lambda x: (x + 255) // 256 * 256
    o_f = r256(d.B * d.H * d.Fc * d.T_pad * d.D * 2) + r256(bhq * d.D * 4)
    o_b = o_f + r256(bhq * max(k_f, 0) * 4)
    o_c = o_b + r256(bhq * max(k_b, 0) * 4)
    raw = ws.cpu().numpy()
    fr = raw[o_f:o_f + bhq * kfe * 4].view(np.int32).reshape(d.B, d.H, d.NQB, kfe)
    bl = raw[o_b:o_b + bhq * k_b * 4].view(np.int32).reshape(d.B, d.H, d.NQB, k_b)
    ct = raw[o_c:o_c + bhq * 4].view(np.int32).reshape(d.B, d.H, d.NQB)
    return fr, bl, ct


def oracle_run(wl, chunk, heads=None, t_begin=0, topp=None, cap=None):
    """Oracle over the window's chunks; returns per-chunk bf16 values and the
    final chunk's path outputs (selection, pooled queries) without attention.
    With ``topp`` the blocks follow the top-p budget with cap ``cap``."""
    H = wl.H if heads is None else len(heads)
    cache = o_path.FrameCache(wl.B, H, wl.D, wl.T_f, wl.blk, wl.window)
    cache.t_begin = t_begin
    centres = key_centres(wl, 0) if wl.keys == "clustered" else None
    t0_cur = wl.t0_of(chunk) + t_begin
    lo = max(t_begin, t0_cur + wl.Fc - wl.window)
    first = (lo - t_begin) // wl.Fc + 1
    hist = []
    for c in range(first, chunk):
        x = inputs(wl, c, 0, heads, centres)
        q, k, v = (bits_to_f64(x[n]) for n in ("q", "k", "v"))
        t0 = wl.t0_of(c) + t_begin
        _, k_rot = o_path.rotate_chunk(q, k, wl.Fh, wl.Fw, wl.Fc, t0, "bf16")
        cache.append(k_rot, v, t0, wl.Fc)
        hist.append((t0, k_rot, x["v"]))
    x = inputs(wl, chunk, 0, heads, centres)
    q, k, v = (bits_to_f64(x[n]) for n in ("q", "k", "v"))
    k_f, k_b = oracle_budget(wl, chunk, t_begin)
    if topp is not None:
        k_b = cap
    out = o_path.run_chunk(cache, q, k, v, Fh=wl.Fh, Fw=wl.Fw, Fc=wl.Fc, t0=t0_cur, k_f=k_f, k_b=k_b,
                           dense=wl.dense, store="bf16", attend_too=False, topp=topp)
    # "hist_t": global indices of the history frames; "hist": the earlier
    # chunks' (t0, rotated K, V bits) for building a GPU cache
    out.update(cache=cache, hist_t=out["hist"], hist=hist, x=x, t0=t0_cur, k_f=k_f, k_b=k_b)
    return out


RNG_SEED = 20260
MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def rope_tol(y64: np.ndarray) -> np.ndarray:
    """RoPE tolerance: 1e-2 absolute, or the bf16 rounding bound of the value
    (half a unit in the last of 8 significant bits, <= 2^-8 |y|) when that is
    larger."""
    return np.maximum(1e-2, np.abs(y64) * 2.0 ** -8 * 1.0001)


__all__ = [n for n in dir() if not n.startswith("_")] + ["WORKLOADS", "math"]


def mutual_best_pairs(frames):
    """Rounds: every unpaired query block names the unpaired block sharing the
    most picked frames (31 or more count as equal), ties to the lower index;
    blocks naming each other pair up; a last lone block pairs with none (-1).
    Pairs in order of their lower block."""
    sets = [set(int(t) for t in f) for f in frames]
    n = len(sets)
    ov = lambda i, j: min(len(sets[i] & sets[j]), 31)
    free, partner = set(range(n)), {}
    while len(free) >= 2:
        best = {}
        for i in free:
            best[i] = max((j for j in free if j != i), key=lambda j: (ov(i, j), -j))
        for i in free:
            if best[i] > i and best[best[i]] == i:
                partner[i], partner[best[i]] = best[i], i
        free -= set(partner)
    return [(i, partner[i]) if i in partner else (i, -1) for i in range(n) if partner.get(i, n) > i]
