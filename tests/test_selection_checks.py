"""CPU checks of the selection validity rule the GPU parity tests apply.

Where two candidates' pooled scores lie within the 1e-5 relative gap of a
top-k cut, the GPU's fp32 ranking may swap them; the parity tests then accept
the GPU's list only if it is still a top-k under the oracle's fp64 scores up
to that gap (tests/_util.py: valid_topk, check_selection). These tests pin
that rule on hand-made scores and on a small oracle run.
"""
import numpy as np

from _util import check_selection, oracle_budget, valid_topk
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
