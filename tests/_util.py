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


def selection_mismatch(gpu_blocks, gpu_cnt, o_blocks, gap_f, gap_b, tol=1e-5):
    """Compare per-(b, h, query block) block lists. Returns (n_units,
    n_mismatch_outside_near_ties, n_near_tie_units)."""
    B, H, NQB, kb = o_blocks.shape
    bad = 0
    near = 0
    for b in range(B):
        for h in range(H):
            for qb in range(NQB):
                same = (gpu_cnt[b, h, qb] == kb and
                        np.array_equal(gpu_blocks[b, h, qb, :kb], o_blocks[b, h, qb]))
                tie = (gap_f[b, h, qb] < tol) or (gap_b[b, h, qb] < tol)
                if tie:
                    near += 1
                elif not same:
                    bad += 1
    return B * H * NQB, bad, near


RNG_SEED = 20260
MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def rope_tol(y64: np.ndarray) -> np.ndarray:
    """RoPE tolerance: 1e-2 absolute, or the bf16 rounding bound of the value
    (half a unit in the last of 8 significant bits, <= 2^-8 |y|) when that is
    larger."""
    return np.maximum(1e-2, np.abs(y64) * 2.0 ** -8 * 1.0001)


__all__ = [n for n in dir() if not n.startswith("_")] + ["WORKLOADS", "math"]
