"""3D rotary position embedding with a global time index (fp64).

Test infrastructure only (see :mod:`oracle`).

Follows "Accelerating Video Generation Inference with Sequential-Parallel 3D
Positional Encoding Using a Global Time Index", section 2B (Causal-RoPE SP):
each chunk starts at a global frame offset ``s`` and a token at local frame
``t`` is rotated with temporal coordinate ``t + s``; the spatial coordinates
(h, w) are the token's row and column inside its frame. Section 2C says the
cos/sin values come from precomputed contiguous tables; the oracle evaluates
them directly in fp64 instead, which is the value the tables approximate.

Readings where the pages are silent:

* pairs are adjacent elements (2p, 2p+1) of the head vector, rotated as a
  complex number;
* the head vector is split into a temporal, a height and a width section,
  in that order; with ``P = D/2`` pairs the height and width sections get
  ``P // 3`` pairs each and the temporal one the rest (D=128: 44/42/42
  dims; D=64: 24/20/20 dims);
* every axis uses base 10000 with the exponent relative to its own section:
  pair j of a section of ``p`` pairs turns at ``10000 ** (-j / p)`` radians
  per unit of position.
"""
from __future__ import annotations

import numpy as np

THETA = 10000.0


def axis_split(D: int):
    """Pairs per axis ``(p_t, p_h, p_w)`` for head dim ``D`` (parity unpinned:
    a reading; the pages give no split)."""
    if D % 2:
        raise ValueError("head_dim must be even")
    P = D // 2
    p_h = P // 3
    return P - 2 * p_h, p_h, p_h


def axis_freqs(p: int, theta: float = THETA) -> np.ndarray:
    """Angular rate of each of an axis's ``p`` pairs: ``theta ** (-2j / (2p))``."""
    j = np.arange(p, dtype=np.float64)
    return theta ** (-(2.0 * j) / (2.0 * p))


def token_coords(Fh: int, Fw: int, Fc: int, t0: int):
    """Global (t, h, w) of every token of a chunk, frame-major then row-major.

    The temporal coordinate is the global time index ``t0 + f`` of local frame
    ``f`` (Causal-RoPE SP, section 2B); h and w restart in every frame.
    """
    n = np.arange(Fc * Fh * Fw)
    T_f = Fh * Fw
    f = n // T_f
    r = n % T_f
    return t0 + f, r // Fw, r % Fw


def pair_angles(D: int, t, h, w, theta: float = THETA) -> np.ndarray:
    """Rotation angle of every (token, pair): ``[n, D/2]`` in fp64."""
    p_t, p_h, p_w = axis_split(D)
    t = np.asarray(t, dtype=np.float64)[:, None]
    h = np.asarray(h, dtype=np.float64)[:, None]
    w = np.asarray(w, dtype=np.float64)[:, None]
    return np.concatenate([t * axis_freqs(p_t, theta)[None, :],
                           h * axis_freqs(p_h, theta)[None, :],
                           w * axis_freqs(p_w, theta)[None, :]], axis=1)


def rotate(x: np.ndarray, angles: np.ndarray) -> np.ndarray:
    """Rotate each pair (x[2p], x[2p+1]) of ``x[..., n, D]`` by ``angles[n, p]``.

    ``y0 = x0 cos - x1 sin``, ``y1 = x0 sin + x1 cos``.
    """
    x = np.asarray(x, dtype=np.float64)
    c = np.cos(angles)
    s = np.sin(angles)
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = x0 * c - x1 * s
    y[..., 1::2] = x0 * s + x1 * c
    return y


def rope_chunk(x: np.ndarray, Fh: int, Fw: int, Fc: int, t0: int,
               theta: float = THETA) -> np.ndarray:
    """Causal-RoPE of one chunk ``x[B, Lq, H, D]`` starting at global frame ``t0``."""
    B, Lq, H, D = x.shape
    t, h, w = token_coords(Fh, Fw, Fc, t0)
    ang = pair_angles(D, t, h, w, theta)                 # [Lq, P]
    xt = np.transpose(np.asarray(x, dtype=np.float64), (0, 2, 1, 3))  # [B,H,Lq,D]
    return np.transpose(rotate(xt, ang), (0, 2, 1, 3))


def tables(D: int, max_t: int, Fh: int, Fw: int, theta: float = THETA):
    """The precomputed cos/sin tables (section 2C), fp64: one ``[positions, pairs]``
    table per axis, in the order t, h, w."""
    p_t, p_h, p_w = axis_split(D)
    out = []
    for n_pos, p in ((max_t, p_t), (Fh, p_h), (Fw, p_w)):
        a = np.arange(n_pos, dtype=np.float64)[:, None] * axis_freqs(p, theta)[None, :]
        out.append((np.cos(a), np.sin(a)))
    return out
