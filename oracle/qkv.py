"""QKV projection followed by Causal-RoPE (fp64).

Test infrastructure only (see :mod:`oracle`).

"Accelerating Video Generation Inference with Sequential-Parallel 3D
Positional Encoding Using a Global Time Index", section 2C (operator
fusion): the QKV projection and the Causal-RoPE computation are merged into
one kernel. What that kernel computes is the projection followed by the
rotation of section 2B, which is what this module states, unfused:

    y = x W^T             x: [B, Lq, C] hidden states of the chunk's tokens,
                          W: [3 H D, C] projection weight
    q, k, v = split(y)    each [B, Lq, H, D]
    q_rot = RoPE(q), k_rot = RoPE(k) with the global time index; v as is.

Readings where the pages are silent:

* the rows of W are the q heads 0..H-1 (D rows each), then the k heads,
  then the v heads (the usual fused-projection layout);
* there is no bias term.
"""
from __future__ import annotations

import numpy as np

from . import rope as _rope


def project(x: np.ndarray, w: np.ndarray, H: int, D: int):
    """``x W^T`` split into q, k, v ``[B, Lq, H, D]`` (fp64)."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    B, Lq, C = x.shape
    if w.shape != (3 * H * D, C):
        raise ValueError("w must be [3*H*D, C]")
    y = x @ w.T                                   # [B, Lq, 3HD]
    y = y.reshape(B, Lq, 3, H, D)
    return y[:, :, 0], y[:, :, 1], y[:, :, 2]


def qkv_rope(x: np.ndarray, w: np.ndarray, H: int, D: int, Fh: int, Fw: int, Fc: int, t0: int):
    """Projection, then Causal-RoPE of q and k for a chunk starting at global
    frame ``t0``. Returns ``q_rot, k_rot, v`` as ``[B, Lq, H, D]`` fp64."""
    q, k, v = project(x, w, H, D)
    return _rope.rope_chunk(q, Fh, Fw, Fc, t0), _rope.rope_chunk(k, Fh, Fw, Fc, t0), v
