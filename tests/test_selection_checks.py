"""CPU checks of the selection validity rule the GPU parity tests apply.

Where two candidates' pooled scores lie within the 1e-5 relative gap of a
top-k cut, the GPU's fp32 ranking may swap them; the parity tests then accept
the GPU's list only if it is still a top-k under the oracle's fp64 scores up
to that gap (tests/_util.py: valid_topk, check_selection). These tests pin
that rule on hand-made scores and on a small oracle run.
"""
import numpy as np

from _util import mutual_best_pairs, check_selection, oracle_budget, valid_topk
from cva_workload import WORKLOADS, chunk_inputs, bf16_bits_to_f32
from oracle import path


def test_valid_topk_accepts_only_swaps_across_a_near_tie():
    s = np.array([3.0, 2.0, 2.0 + 1e-7, 1.0, 0.5])
    assert valid_topk(s, [0, 2], 2, 1e-5)          # exact top-2
    assert valid_topk(s, [0, 1], 2, 1e-5)          # 2.0 and 2.0+1e-7 swap
    assert not valid_topk(s, [0, 3], 2, 1e-5)      # 1.0 is far below the cut
    assert not valid_topk(s, [1, 2], 2, 1e-5)      # 3.0 must be taken
    assert not valid_topk(s, [0, 0], 2, 1e-5)      # duplicates
    assert not valid_topk(s, [0], 2, 1e-5)         # wrong count
    assert valid_topk(s, [0, 1, 2, 3, 4], 5, 1e-5)  # everything
    far = np.array([3.0, 2.0, 1.0])
    assert not valid_topk(far, [0, 2], 2, 1e-5)    # no tie: only the exact set


def _small_run():
    wl = WORKLOADS["r64"]
    cache = path.FrameCache(wl.B, wl.H, wl.D, wl.T_f, wl.blk, wl.window)
    out = None
    for c in range(1, wl.chunk + 1):
        x = chunk_inputs(wl, c, 0)
        q, k, v = (bf16_bits_to_f32(x[n]).astype(np.float64) for n in ("q", "k", "v"))
        k_f, k_b = oracle_budget(wl, c)
        out = path.run_chunk(cache, q, k, v, Fh=wl.Fh, Fw=wl.Fw, Fc=wl.Fc, t0=wl.t0_of(c),
                             k_f=k_f, k_b=k_b, dense=False, attend_too=False)
    out["cache"] = cache
    return out


def test_check_selection_counts_wrong_lists_and_substitutes_valid_ones():
    run = _small_run()
    fr, bl = run["frames"].copy(), run["blocks"].copy()
    cnt = np.full(bl.shape[:-1], bl.shape[-1])
    n, bad, near, blocks = check_selection(run, fr, bl, cnt)
    assert (bad, near) == (0, 0)
    np.testing.assert_array_equal(blocks, run["blocks"])
    # a list that swaps a picked block for an unpicked one of the same frames is wrong
    nb = run["cache"].nb
    b, h, qb = 0, 1, 2
    cand = set((fr[b, h, qb][:, None] * nb + np.arange(nb)[None, :]).reshape(-1).tolist())
    other = sorted(cand - set(bl[b, h, qb].tolist()))
    assert other, "the small case must leave an unpicked candidate"
    wrong = bl.copy()
    wrong[b, h, qb, 0] = other[0]
    wrong[b, h, qb] = np.sort(wrong[b, h, qb])
    n, bad, near, _ = check_selection(run, fr, wrong, cnt)
    assert bad == 1 and near == 0
    # a wrong count is wrong too
    c2 = cnt.copy()
    c2[b, h, qb] -= 1
    assert check_selection(run, fr, bl, c2)[1] == 1
    # a frame list that is not a top-k of the frame scores is wrong
    hist = np.asarray(run["hist"])
    if len(hist) > fr.shape[-1]:
        unpicked = sorted(set(hist.tolist()) - set(fr[b, h, qb].tolist()))
        f2 = fr.copy()
        f2[b, h, qb, 0] = unpicked[0]
        f2[b, h, qb] = np.sort(f2[b, h, qb])
        assert check_selection(run, f2, bl, cnt)[1] >= 1


def test_mutual_best_pairs_by_hand():
    # frame sets of 5 query blocks: 0 and 3 share three frames, 1 and 2 two,
    # 4 shares at most one with anyone: round 1 pairs (0, 3) and (1, 2); block
    # 4 is left alone
    frames = [[0, 1, 2], [5, 6, 7], [5, 6, 9], [0, 1, 2], [2, 9, 11]]
    assert mutual_best_pairs(frames) == [(0, 3), (1, 2), (4, -1)]
    # ties go to the lower index: 1, 2 and 3 all share one frame with 0
    frames = [[0, 1], [0, 5], [0, 6], [0, 7]]
    assert mutual_best_pairs(frames) == [(0, 1), (2, 3)]


def test_mutual_best_pairs_partition_and_round_rule():
    rng = np.random.default_rng(7)
    for trial in range(40):
        n = int(rng.integers(1, 40))
        F, k = int(rng.integers(2, 20)), None
        k = int(rng.integers(1, F + 1))
        frames = [sorted(rng.choice(F, size=k, replace=False).tolist()) for _ in range(n)]
        pairs = mutual_best_pairs(frames)
        ids = sorted(v for p in pairs for v in p if v >= 0)
        assert ids == list(range(n))                              # a partition
        assert [p[0] for p in pairs] == sorted(p[0] for p in pairs)
        assert all(j == -1 or i < j for i, j in pairs)
        assert sum(1 for _, j in pairs if j == -1) == n % 2     # one lone block at most
        # the best pair overall (most shared frames, then lowest indices) is always formed
        if n >= 2:
            sets = [set(f) for f in frames]
            ov = lambda i, j: min(len(sets[i] & sets[j]), 31)
            top = max(((ov(i, j), -i, -j) for i in range(n) for j in range(i + 1, n)))
            assert (-top[1], -top[2]) in pairs
