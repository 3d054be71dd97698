"""Attention over an explicit key set (fp64).

Test infrastructure only (see :mod:`oracle`).

Follows "Light Forcing", section 2.2 (execution): attention is computed only
over the picked frame-block pairs, here together with every token of the
current chunk (queries see earlier chunks and their own chunk, the causal
chunk-by-chunk generation of "Accelerating Video Generation Inference ...",
section 1). Within the key set the softmax is the ordinary one with scale
``1/sqrt(D)`` (a reading: the pages print no scale).
"""
from __future__ import annotations

import numpy as np


def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """``o_i = sum_j softmax_j(scale * q_i . k_j) v_j`` and ``lse_i`` (natural log).

    Two passes: the row maximum first, then the exponentials shifted by it.
    ``q[nq, D]``, ``k[nk, D]``, ``v[nk, D]``; ``nk`` must be positive.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if k.shape[0] == 0:
        raise ValueError("empty key set")
    s = (q @ k.T) * scale
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    o = (p @ v) / l
    return o, (m + np.log(l))[:, 0]
