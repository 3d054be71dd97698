"""Seeded synthetic workloads for the per-chunk attention path.

This module only *describes* and *draws* inputs. It holds none of the
method's arithmetic (no rotary embedding, pooling, selection, attention or
budget rule): both the CUDA library's tests and the fp64 oracle consume what
it produces, so it must stay neutral.

Shapes follow the Wan2.1-shaped workloads of the streaming video DiT pages
(480P latent grid 30x52, 720P latent grid 45x80, three latent frames per
chunk) and a tiny 8x8 case. Inputs are drawn with numpy's PCG64 generator,
in float32, and rounded once to bfloat16 (round to nearest even); the
rounded bits are what both sides consume.

Token order inside a chunk is frame-major, then row-major (h, w) inside a
frame. Tensors are laid out ``[B, Lq, H, D]`` (the order a QKV projection
emits them).
"""
from __future__ import annotations

import dataclasses
from fractions import Fraction
from typing import Dict, Optional

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "seed_for", "bf16_bits", "bf16_bits_to_f32",
    "chunk_inputs", "key_centres",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload.

    ``chunk`` is the 1-based index of the chunk that is timed or checked; its
    global start frame is ``t0 = Fc * (chunk - 1)`` and every earlier chunk
    of the same layer is its history (frames ``0 .. t0-1``), of which a
    rolling cache of ``window`` frame slots keeps the newest.

    The selection budget is data here, not a rule: ``k_f_max`` frames and a
    key density ``d_i = d_base + d_slope * (i - d_pivot)`` over the history
    blocks, as exact rationals. ``dense=True`` selects everything.
    """
    key: str
    name: str
    config_index: int
    B: int
    H: int
    D: int
    Fh: int
    Fw: int
    Fc: int
    blk: int
    window: int
    chunk: int
    keys: str = "normal"          # "normal" or "clustered"
    dense: bool = True
    k_f_max: int = 0
    d_base: Fraction = Fraction(0)
    d_slope: Fraction = Fraction(0)
    d_pivot: int = 0
    k_b_fixed: Optional[int] = None   # a fixed block count instead of a density
    layers: int = 1
    chunks: int = 1               # streaming runs walk chunks 1..chunks
    input_dtype: str = "bf16"     # "fp32": drawn fp32, rounded to bf16 once
    centres: int = 16
    sigma: float = 0.3

    # derived sizes -------------------------------------------------------
    @property
    def T_f(self) -> int:
        return self.Fh * self.Fw

    @property
    def nb(self) -> int:
        return -(-self.T_f // self.blk)

    @property
    def T_pad(self) -> int:
        return self.nb * self.blk

    @property
    def Lq(self) -> int:
        return self.Fc * self.T_f

    @property
    def NQB(self) -> int:
        return self.Fc * self.nb

    @property
    def t0(self) -> int:
        return self.Fc * (self.chunk - 1)

    def t0_of(self, chunk: int) -> int:
        return self.Fc * (chunk - 1)

    def with_chunk(self, chunk: int) -> "Workload":
        return dataclasses.replace(self, chunk=chunk)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _wl(**kw) -> Workload:
    return Workload(**kw)


WORKLOADS: Dict[str, Workload] = {
    # Tiny case: 8x8 grid, 3-frame chunk, 9 history frames (chunk 4, t0=9).
    "c1": _wl(key="c1", name="tiny-8x8-d64", config_index=1, B=1, H=2, D=64,
              Fh=8, Fw=8, Fc=3, blk=64, window=12, chunk=4,
              input_dtype="fp32", dense=True),
    "c1s": _wl(key="c1s", name="tiny-8x8-d64-sparse", config_index=1, B=1,
               H=2, D=64, Fh=8, Fw=8, Fc=3, blk=64, window=12, chunk=4,
               input_dtype="fp32", dense=False, k_f_max=4, k_b_fixed=4),
    # Wan-1.3B shaped dense layer: 18 history frames + the chunk.
    "c2": _wl(key="c2", name="wan1.3b-480p-dense", config_index=2, B=1,
              H=12, D=128, Fh=30, Fw=52, Fc=3, blk=64, window=21, chunk=7,
              dense=True),
    # Same shape, clustered keys, hierarchical selection, chunk-aware budget
    # d_i = 1/4 + (i-6)/60 (the schedule read literally; chunk 1 is dense).
    "c3": _wl(key="c3", name="wan1.3b-480p-hsa", config_index=3, B=1, H=12,
              D=128, Fh=30, Fw=52, Fc=3, blk=64, window=21, chunk=7,
              keys="clustered", dense=False, k_f_max=8,
              d_base=Fraction(1, 4), d_slope=Fraction(1, 60), d_pivot=6,
              chunks=7),
    # 14B-shaped 720P layer, block 128, top-6 frames, 20% block density.
    "c4": _wl(key="c4", name="wan14b-720p-hsa", config_index=4, B=1, H=40,
              D=128, Fh=45, Fw=80, Fc=3, blk=128, window=21, chunk=7,
              keys="clustered", dense=False, k_f_max=6,
              d_base=Fraction(1, 5)),
    # Streaming: 80 chunks x 30 layers, rolling window of 60 frame slots.
    "c5": _wl(key="c5", name="wan1.3b-480p-stream", config_index=5, B=1,
              H=12, D=128, Fh=30, Fw=52, Fc=3, blk=64, window=60, chunk=80,
              keys="clustered", dense=False, k_f_max=20,
              d_base=Fraction(1, 5), layers=30, chunks=80),
    # Small parity cases with ragged frame tails (not in the pages' list):
    # 120 tokens per frame over 64-token blocks (tail 56) and 200 tokens
    # per frame over 128-token blocks (tail 72).
    "r64": _wl(key="r64", name="ragged-6x20-b64", config_index=6, B=1, H=2,
               D=128, Fh=6, Fw=20, Fc=3, blk=64, window=9, chunk=3,
               keys="clustered", dense=False, k_f_max=4,
               d_base=Fraction(1, 2)),
    "r128": _wl(key="r128", name="ragged-10x20-b128", config_index=7, B=2,
                H=3, D=128, Fh=10, Fw=20, Fc=3, blk=128, window=12, chunk=4,
                keys="clustered", dense=False, k_f_max=3,
                d_base=Fraction(1, 4)),
    "r64s": _wl(key="r64s", name="ragged-5x9-d64", config_index=8, B=2,
                H=2, D=64, Fh=5, Fw=9, Fc=3, blk=64, window=8, chunk=5,
                keys="clustered", dense=False, k_f_max=3,
                d_base=Fraction(2, 5)),
}


def seed_for(config_index: int, chunk: int, layer: int) -> int:
    """Seed of one (config, chunk, layer) draw: 1e6*config + 1e3*chunk + layer."""
    return 1_000_000 * config_index + 1_000 * chunk + layer


# --- bfloat16 storage helpers (input preparation only) -------------------

def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return the bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bits to float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


# --- draws -----------------------------------------------------------------

def key_centres(wl: Workload, layer: int = 0) -> np.ndarray:
    """Per-head cluster centres ``[H, centres, D]`` ~ N(0, I), fixed per layer."""
    rng = np.random.Generator(np.random.PCG64(seed_for(wl.config_index, 0, layer)))
    return rng.standard_normal((wl.H, wl.centres, wl.D), dtype=np.float32)


def chunk_inputs(wl: Workload, chunk: Optional[int] = None, layer: int = 0,
                 centres: Optional[np.ndarray] = None) -> dict:
    """Raw Q, K, V of one chunk, ``[B, Lq, H, D]``.

    Returns a dict with float32 ``q32/k32/v32`` (the draws) and ``q/k/v``,
    the bfloat16 bits (uint16) both sides consume.

    Clustered keys: each (batch, head, frame, key block) picks one of the
    head's centres uniformly, and its tokens are ``centre + sigma * N(0, I)``.
    Q and V are N(0, 1).
    """
    c = wl.chunk if chunk is None else chunk
    rng = np.random.Generator(np.random.PCG64(seed_for(wl.config_index, c, layer)))
    shape = (wl.B, wl.Lq, wl.H, wl.D)
    z = None
    if wl.keys == "clustered":
        if centres is None:
            centres = key_centres(wl, layer)
        z = rng.integers(0, wl.centres, size=(wl.B, wl.H, wl.Fc, wl.nb))
    q32 = rng.standard_normal(shape, dtype=np.float32)
    noise = rng.standard_normal(shape, dtype=np.float32)
    v32 = rng.standard_normal(shape, dtype=np.float32)
    if z is None:
        k32 = noise
    else:
        # token n of frame f, row r -> key block r // blk
        n = np.arange(wl.Lq)
        f = n // wl.T_f
        j = (n % wl.T_f) // wl.blk
        zz = z[:, :, f, j]                                   # [B, H, Lq]
        h_idx = np.arange(wl.H)[None, :, None]
        mu = centres[h_idx, zz]                              # [B, H, Lq, D]
        k32 = np.transpose(mu, (0, 2, 1, 3)) + np.float32(wl.sigma) * noise
        k32 = k32.astype(np.float32)
    return {
        "q32": q32, "k32": k32, "v32": v32,
        "q": bf16_bits(q32), "k": bf16_bits(k32), "v": bf16_bits(v32),
        "chunk": c, "layer": layer, "t0": wl.t0_of(c),
    }


def hidden_inputs(wl: Workload, hidden: int, chunk: Optional[int] = None, layer: int = 0) -> dict:
    """Hidden states of one chunk and a projection weight for the fused QKV
    step: ``x [B, Lq, C]`` N(0, 1) and ``w [3 H D, C]`` N(0, 1/C) (so the
    projected q, k, v are about N(0, 1)), drawn in fp32 from the chunk's
    seed (offset so they differ from :func:`chunk_inputs`) and rounded once
    to bfloat16. Returns the bits (uint16) under ``x`` and ``w``."""
    c = wl.chunk if chunk is None else chunk
    rng = np.random.Generator(np.random.PCG64(seed_for(wl.config_index, c, layer) + 500))
    x32 = rng.standard_normal((wl.B, wl.Lq, hidden), dtype=np.float32)
    w32 = rng.standard_normal((3 * wl.H * wl.D, hidden), dtype=np.float32) / np.float32(np.sqrt(hidden))
    return {"x": bf16_bits(x32), "w": bf16_bits(w32)}
