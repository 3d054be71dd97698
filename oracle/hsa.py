"""Hierarchical sparse selection and the chunk budget (fp64).

Test infrastructure only (see :mod:`oracle`).

Follows "Light Forcing":

* section 2.2, token compression: query and key tokens are mean-pooled per
  block and per frame (:func:`block_means`, :func:`frame_mean`);
* section 2.2, two-level selection: for each query block, a few history
  frames are picked with the frame-pooled keys (:func:`frame_select`), then
  the important blocks inside those frames with the block-pooled keys
  (:func:`block_select`);
* section 2.1, Chunk-Aware Growth: the budget is set per chunk, the first
  chunk dense (:func:`budget`).

Readings where the pages are silent: blocks are per frame (the last block
of a frame holds the remainder); pooling is applied to the rotated Q and K;
the frame-pooled key is the token mean of the frame; the query that drives
both levels is the block-pooled query of that query block; scores are raw
dot products; ties go to the lower global frame index, then the lower block
index; ``k_b`` counts blocks over all picked frames together; the chosen
blocks are reported in ascending (frame, block) order as ``t * nb + j``.
"""
from __future__ import annotations

import math
from fractions import Fraction
from typing import Optional, Tuple

import numpy as np


# --- pooling -----------------------------------------------------------------

def block_means(x: np.ndarray, blk: int) -> np.ndarray:
    """Mean over each block's valid tokens: ``x[..., T_f, D] -> [..., nb, D]``.

    Block j of a frame holds tokens ``[j*blk, min((j+1)*blk, T_f))``.
    """
    T_f = x.shape[-2]
    nb = -(-T_f // blk)
    out = [np.asarray(x[..., j * blk:min((j + 1) * blk, T_f), :],
                      dtype=np.float64).mean(axis=-2) for j in range(nb)]
    return np.stack(out, axis=-2)


def frame_mean(x: np.ndarray) -> np.ndarray:
    """Token mean of a whole frame: ``x[..., T_f, D] -> [..., D]``."""
    return np.asarray(x, dtype=np.float64).mean(axis=-2)


# --- selection -----------------------------------------------------------------

def rel_gap(a: float, b: float) -> float:
    """``|a - b| / max(|a|, |b|, 1e-30)``: how far a top-k boundary is from a tie."""
    return abs(a - b) / max(abs(a), abs(b), 1e-30)


def topk(scores: np.ndarray, k: int) -> Tuple[np.ndarray, float]:
    """Positions of the ``k`` largest scores, ties to the lower position.

    Returns the chosen positions in ascending order and the relative gap
    between the k-th and (k+1)-th score in rank order (``inf`` when all are
    taken).
    """
    scores = np.asarray(scores, dtype=np.float64)
    n = scores.shape[0]
    if k < 0 or k > n:
        raise ValueError("k out of range")
    order = np.lexsort((np.arange(n), -scores))          # by -score, then position
    chosen = np.sort(order[:k])
    gap = math.inf if (k == n or k == 0) else rel_gap(scores[order[k - 1]], scores[order[k]])
    return chosen, gap


def frame_select(qbar: np.ndarray, kbar_frames: np.ndarray, frame_t: np.ndarray,
                 k_f: int) -> Tuple[np.ndarray, float]:
    """First level: pick ``k_f`` history frames for one query block.

    ``qbar[D]`` is the block-pooled query (parity unpinned: the pages say
    "for each query block" but not which pooled query scores the frames),
    ``kbar_frames[F, D]`` the frame-pooled keys of the history frames whose
    global indices are ``frame_t[F]`` (ascending). With ``F <= k_f`` every
    frame is kept. Returns the chosen global frame indices (ascending) and
    the boundary gap.
    """
    frame_t = np.asarray(frame_t)
    F = frame_t.shape[0]
    if F <= k_f:
        return frame_t.copy(), math.inf
    scores = kbar_frames @ np.asarray(qbar, dtype=np.float64)
    pos, gap = topk(scores, k_f)
    return frame_t[pos], gap


def block_select(qbar: np.ndarray, kbar_blocks: np.ndarray, frames_t: np.ndarray,
                 nb: int, k_b: int) -> Tuple[np.ndarray, float]:
    """Second level: pick ``k_b`` blocks among all blocks of the picked frames.

    ``kbar_blocks[F_sel, nb, D]`` are the block-pooled keys of the picked frames
    ``frames_t`` (ascending). Candidates are enumerated in ascending (t, j)
    order, so "lower position" is "lower frame, then lower block". Returns the
    chosen ids ``t * nb + j`` (ascending) and the boundary gap.
    """
    frames_t = np.asarray(frames_t)
    cand_scores = (kbar_blocks.reshape(-1, kbar_blocks.shape[-1])
                   @ np.asarray(qbar, dtype=np.float64))
    cand_ids = (frames_t[:, None] * nb + np.arange(nb)[None, :]).reshape(-1)
    pos, gap = topk(cand_scores, k_b)
    return cand_ids[pos], gap


def topp_ranking(qbar: np.ndarray, kbar_blocks: np.ndarray, frames_t: np.ndarray,
                 nb: int, T_f: int, blk: int):
    """Candidate blocks of the picked frames in rank order, for the top-p budget.

    Returns ``(ids, scores, above)`` in rank order (score descending, ties to
    the lower position): the ids ``t * nb + j``, the pooled scores and the
    share of the estimated attention ranked above each candidate (see
    :func:`block_select_topp`).
    """
    frames_t = np.asarray(frames_t)
    qbar = np.asarray(qbar, dtype=np.float64)
    D = qbar.shape[0]
    s = kbar_blocks.reshape(-1, kbar_blocks.shape[-1]) @ qbar
    C = s.shape[0]
    cand_ids = (frames_t[:, None] * nb + np.arange(nb)[None, :]).reshape(-1)
    tail = T_f - (nb - 1) * blk
    n = np.tile(np.array([blk] * (nb - 1) + [tail], dtype=np.float64), frames_t.shape[0])
    order = np.lexsort((np.arange(C), -s))
    m = n * np.exp((s - s.max()) / math.sqrt(D))
    ms = m[order]
    above = (np.cumsum(ms) - ms) / m.sum()
    return cand_ids[order], s[order], above


def block_select_topp(qbar: np.ndarray, kbar_blocks: np.ndarray, frames_t: np.ndarray,
                      nb: int, T_f: int, blk: int, p: float, k_cap: int):
    """Second level with a top-p budget instead of a fixed ``k_b``.

    "Sparse VideoGen2", section B (centroid top-p): clusters are sorted by
    their estimated attention scores and taken one after another until the
    cumulative score reaches the threshold ``p``. Readings for key blocks:

    * the candidates are the blocks of the picked frames, ranked as in
      :func:`block_select` (pooled score ``q.kb``, ties to the lower
      position);
    * a block's estimated attention is its share of the softmax of the
      pooled scores weighted by its valid token count,
      ``m_c = n_c exp(s_c / sqrt(D)) / sum_c' n_c' exp(s_c' / sqrt(D))``;
    * the shortest prefix of the ranking whose mass reaches ``p`` is taken:
      block c goes in when the mass ranked above it is below ``p``; at least
      one block, at most ``k_cap`` (the list size).

    Returns the chosen ids ``t * nb + j`` (ascending) and a boundary gap: the
    smallest of the relative score gap at the cut and the distance of the
    threshold from the cumulative masses around the cut (``inf`` when no
    candidate was left out).
    """
    ids, s, above = topp_ranking(qbar, kbar_blocks, frames_t, nb, T_f, blk)
    C = ids.shape[0]
    take = (above < p) & (np.arange(C) < k_cap)
    take[0] = k_cap > 0                                    # at least one block
    r = int(take.sum())
    gap = math.inf
    if r < C:
        gap = min(rel_gap(s[r - 1], s[r]) if r > 0 else math.inf,
                  abs(above[r] - p), abs(above[r - 1] - p) if r > 0 else math.inf)
    return np.sort(ids[:r]), gap


# --- chunk budget -----------------------------------------------------------------

def density(d_base: Fraction, d_slope: Fraction, d_pivot: int, chunk: int) -> Fraction:
    """Key density of chunk ``i``: ``d_base + d_slope * (i - pivot)``, clamped to [0, 1].

    With the schedule read literally (sparsity ``s_i = 3/4 - (i - 6)/60``),
    density is ``1 - s_i = 1/4 + (i - 6)/60`` (parity unpinned: the pages
    state the opposite direction in words; the schedule is a parameter).
    """
    d = Fraction(d_base) + Fraction(d_slope) * (chunk - d_pivot)
    return min(max(d, Fraction(0)), Fraction(1))


def budget(chunk: int, hist_frames: int, nb: int, *, dense: bool, k_f_max: int,
           d_base: Fraction = Fraction(0), d_slope: Fraction = Fraction(0),
           d_pivot: int = 0, k_b_fixed: Optional[int] = None) -> Tuple[int, int]:
    """``(k_f, k_b)`` of one chunk (Light Forcing section 2.1).

    The first chunk, and every chunk when ``dense``, keeps all history.
    Otherwise ``k_f = min(k_f_max, hist_frames)`` and ``k_b`` is the density
    times the number of history blocks, rounded half up, at most the number
    of candidate blocks ``k_f * nb`` (or ``k_b_fixed`` when given).
    """
    all_blocks = hist_frames * nb
    if dense or chunk <= 1 or hist_frames == 0:
        return hist_frames, all_blocks
    k_f = min(k_f_max, hist_frames)
    cand = k_f * nb
    if k_b_fixed is not None:
        return k_f, min(cand, int(k_b_fixed))
    d = density(d_base, d_slope, d_pivot, chunk)
    k_b = math.floor(d * all_blocks + Fraction(1, 2))
    return k_f, min(cand, k_b)


# --- chunk budget from the noise level (Light Forcing section 2.1) -------------------

NOISE_BISECTION_STEPS = 200


def noise_densities(n_chunks: int, Fc: int, window: int, nb: int, s_base: float, s_target: float):
    """Key density of chunks 2..n from ``s_i = s_base - alpha_i * beta``.

    Light Forcing, section 2.1: ``alpha_i`` scales with the noise level as
    ``1/sqrt(T)`` and ``beta`` is set so that the total attention FLOPs meet
    a target sparsity. Readings (the pages garble the formula):

    * the noise level of chunk ``i`` grows with its index in the chunk
      schedule, ``alpha_i = 1 / sqrt(i)``, so later chunks get more sparsity;
    * density is ``d_i = 1 - s_i``, clamped to [0, 1], and counts history
      blocks (the current chunk is always dense);
    * the FLOP target is ``sum_i d_i N_i = (1 - s_target) sum_i N_i`` over
      chunks 2..n, with ``N_i`` the history blocks of chunk ``i`` in a
      rolling window of ``window`` frames;
    * ``beta`` is found by bisection on [-2^20, 2^20] (the sum grows with
      beta) in a fixed number of fp64 steps, the same in the library.

    Returns ``{i: d_i}`` for i = 2..n (chunk 1 is dense).
    """
    chunks = list(range(2, n_chunks + 1))
    N = {i: min(Fc * (i - 1), window - Fc) * nb for i in chunks}
    alpha = {i: 1.0 / math.sqrt(i) for i in chunks}
    d0 = 1.0 - s_base
    goal = (1.0 - s_target) * sum(N[i] for i in chunks)

    def dens(i, beta):
        return min(max(d0 + alpha[i] * beta, 0.0), 1.0)

    def total(beta):
        s = 0.0
        for i in chunks:
            s += dens(i, beta) * N[i]
        return s

    lo, hi = -1048576.0, 1048576.0
    for _ in range(NOISE_BISECTION_STEPS):
        mid = 0.5 * (lo + hi)
        if total(mid) < goal:
            lo = mid
        else:
            hi = mid
    return {i: dens(i, hi) for i in chunks}


def noise_budget(chunk: int, hist_frames: int, nb: int, k_f_max: int, density_i: float) -> Tuple[int, int]:
    """``(k_f, k_b)`` of a chunk with a given density: ``k_f = min(k_f_max,
    history)`` and ``k_b = floor(d * history blocks + 1/2)`` at most the
    candidates ``k_f * nb`` (as :func:`budget`, in fp64 for the density)."""
    all_blocks = hist_frames * nb
    if chunk <= 1 or hist_frames == 0:
        return hist_frames, all_blocks
    k_f = min(k_f_max, hist_frames)
    return k_f, min(k_f * nb, int(math.floor(density_i * all_blocks + 0.5)))
