"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each test checks the oracle against mathematics, a closed form, a library
routine or brute force on tiny inputs, chosen so that a plausible slip (a
dropped term, a wrong sign, a swapped axis, an off-by-one in a block edge, a
wrong tie-break) fails at least one of them.
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest
import scipy.special

from oracle import rope, hsa, path
from oracle.attention import attend
from cva_workload import WORKLOADS, chunk_inputs, bf16_bits_to_f32


RNG = np.random.default_rng(1234)


# --- RoPE ------------------------------------------------------------------

def _rot(x, t, h, w):
    x = np.asarray(x, dtype=np.float64)
    ang = rope.pair_angles(x.shape[-1], np.atleast_1d(t), np.atleast_1d(h), np.atleast_1d(w))
    return rope.rotate(x[None, :], ang)[0]


def test_rope_closed_form_d6():
    # D=6: one pair per axis, every rate is 10000**0 = 1, so the angles are the
    # positions themselves.
    x = np.array([1.0, 0.0, 0.0, 1.0, 1.0, 1.0])
    y = _rot(x, 1, 2, 3)
    c, s = math.cos, math.sin
    want = [c(1), s(1), -s(2), c(2), c(3) - s(3), s(3) + c(3)]
    np.testing.assert_allclose(y, want, rtol=0, atol=1e-15)


def test_axis_split_matches_wan_sections():
    # 128 -> 44/42/42 dims, 64 -> 24/20/20 dims (pairs 22/21/21 and 12/10/10).
    assert rope.axis_split(128) == (22, 21, 21)
    assert rope.axis_split(64) == (12, 10, 10)


def test_rope_rates_first_and_last_pair():
    # pair j of an axis with p pairs turns at 10000**(-j/p) rad per position
    for p in (10, 12, 21, 22):
        f = rope.axis_freqs(p)
        assert f[0] == 1.0
        assert f[-1] == pytest.approx(10000.0 ** (-(p - 1) / p), rel=1e-15)
        assert np.all(np.diff(f) < 0)


@pytest.mark.parametrize("D", [64, 128])
def test_rope_norm_preserved(D):
    x = RNG.standard_normal((50, D))
    t, h, w = RNG.integers(0, 300, 50), RNG.integers(0, 45, 50), RNG.integers(0, 80, 50)
    y = rope.rotate(x, rope.pair_angles(D, t, h, w))
    nx = x[:, 0::2] ** 2 + x[:, 1::2] ** 2
    ny = y[:, 0::2] ** 2 + y[:, 1::2] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("D", [64, 128])
def test_rope_relative_position(D):
    # <R(m) q, R(n) k> == <q, R(n - m) k>: scores depend on the offset only.
    for _ in range(20):
        q, k = RNG.standard_normal(D), RNG.standard_normal(D)
        m = RNG.integers(0, 200, 3)
        n = RNG.integers(0, 200, 3)
        lhs = _rot(q, *m) @ _rot(k, *n)
        rhs = q @ _rot(k, *(n - m))
        assert lhs == pytest.approx(rhs, rel=1e-11, abs=1e-11)


def test_rope_position_zero_is_identity():
    x = RNG.standard_normal((4, 128))
    y = rope.rotate(x, rope.pair_angles(128, [0] * 4, [0] * 4, [0] * 4))
    np.testing.assert_array_equal(y, x)


def test_rope_axis_sections_in_order_t_h_w():
    # A coordinate on one axis only moves that axis's section of the vector.
    D = 128
    p_t, p_h, p_w = rope.axis_split(D)
    x = RNG.standard_normal(D)
    sec = {"t": slice(0, 2 * p_t), "h": slice(2 * p_t, 2 * (p_t + p_h)),
           "w": slice(2 * (p_t + p_h), D)}
    for axis, pos in (("t", (5, 0, 0)), ("h", (0, 5, 0)), ("w", (0, 0, 5))):
        y = _rot(x, *pos)
        for other, sl in sec.items():
            if other == axis:
                assert not np.allclose(y[sl], x[sl])
            else:
                np.testing.assert_array_equal(y[sl], x[sl])


def test_rope_complex_restatement():
    # (x0 + i x1) * exp(i phi) with phi built from the pages' t = t0 + f rule.
    D, Fh, Fw, Fc, t0 = 64, 3, 4, 2, 7
    x = RNG.standard_normal((1, Fc * Fh * Fw, 1, D))
    y = rope.rope_chunk(x, Fh, Fw, Fc, t0)[0, :, 0]
    z = x[0, :, 0, 0::2] + 1j * x[0, :, 0, 1::2]
    p_t, p_h, p_w = rope.axis_split(D)
    for n in range(Fc * Fh * Fw):
        f, r = divmod(n, Fh * Fw)
        hh, ww = divmod(r, Fw)
        phi = np.concatenate([(t0 + f) * 10000.0 ** (-np.arange(p_t) / p_t),
                              hh * 10000.0 ** (-np.arange(p_h) / p_h),
                              ww * 10000.0 ** (-np.arange(p_w) / p_w)])
        zz = z[n] * np.exp(1j * phi)
        np.testing.assert_allclose(y[n, 0::2], zz.real, atol=1e-12)
        np.testing.assert_allclose(y[n, 1::2], zz.imag, atol=1e-12)


def test_global_time_index_tokens():
    # token n of a chunk starting at s has global t = s + n // T_f
    t, h, w = rope.token_coords(3, 5, 3, 42)
    assert list(t[:15]) == [42] * 15 and list(t[15:30]) == [43] * 15 and t[-1] == 44
    assert h[7] == 1 and w[7] == 2


def test_tables_match_direct_angles():
    (ct, st), (ch, sh), (cw, sw) = rope.tables(128, 240, 30, 52)
    assert ct.shape == (240, 22) and ch.shape == (30, 21) and cw.shape == (52, 21)
    ang = rope.pair_angles(128, [239], [29], [51])[0]
    np.testing.assert_allclose(ct[239], np.cos(ang[:22]), atol=1e-15)
    np.testing.assert_allclose(sw[51], np.sin(ang[43:]), atol=1e-15)


# --- bf16 rounding ------------------------------------------------------------

def test_round_bf16_matches_bit_rounding_of_float32():
    # For float32-representable inputs the exact rounding equals rounding the
    # float32 bit pattern (a different construction).
    from cva_workload import bf16_bits
    x = RNG.standard_normal(100000).astype(np.float32) * np.float32(3.0)
    x[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -0.0, 2 ** -130]   # ties and a subnormal
    want = bf16_bits_to_f32(bf16_bits(x)).astype(np.float64)
    got = path.round_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(got, want)


# --- pooling ------------------------------------------------------------------

def test_block_means_ragged_tail_and_weighted_frame_mean():
    x = RNG.standard_normal((2, 1560, 8))
    bm = hsa.block_means(x, 64)
    assert bm.shape == (2, 25, 8)
    # library mean of the explicit slices, including the 24-token tail
    np.testing.assert_allclose(bm[:, 24], np.mean(x[:, 1536:1560], axis=1), rtol=1e-13)
    np.testing.assert_allclose(bm[:, 3], np.mean(x[:, 192:256], axis=1), rtol=1e-13)
    counts = np.array([64] * 24 + [24])
    fm = np.average(bm, axis=1, weights=counts)
    np.testing.assert_allclose(hsa.frame_mean(x), fm, rtol=1e-12, atol=1e-15)
    # the frame mean is a token mean, not a mean of block means
    assert not np.allclose(hsa.frame_mean(x), bm.mean(axis=1))


def test_pool_queries_layout():
    B, H, D, Fh, Fw, Fc, blk = 1, 2, 4, 3, 5, 2, 8
    q = RNG.standard_normal((B, Fc * Fh * Fw, H, D))
    qb, qf = path.pool_queries(q, Fh * Fw, blk, Fc)
    assert qb.shape == (B, H, Fc * 2, D)
    # query block 3 = frame 1, block 1 = tokens 15+8 .. 15+14
    np.testing.assert_allclose(qb[0, 1, 3], q[0, 23:30, 1].mean(0), rtol=1e-13)
    np.testing.assert_allclose(qf[0, 0, 1], q[0, 15:30, 0].mean(0), rtol=1e-13)


# --- selection ----------------------------------------------------------------

def _brute_topk(scores, k):
    best = None
    for sub in itertools.combinations(range(len(scores)), k):
        key = (sum(scores[i] for i in sub), [-i for i in sub])
        if best is None or key > best[0]:
            best = (key, sub)
    return np.array(best[1])


def test_topk_equals_brute_force_with_ties():
    for trial in range(60):
        n = int(RNG.integers(1, 10))
        k = int(RNG.integers(0, n + 1))
        # small integer scores force ties
        s = RNG.integers(-3, 4, n).astype(np.float64)
        got, _ = hsa.topk(s, k)
        np.testing.assert_array_equal(got, _brute_topk(list(s), k))


def test_topk_tie_goes_to_lower_index():
    got, gap = hsa.topk(np.array([1.0, 2.0, 2.0, 2.0, 0.5]), 2)
    assert list(got) == [1, 2] and gap == 0.0


def test_block_select_ids_and_full_budget():
    nb, D = 3, 4
    frames = np.array([2, 5])
    kb = RNG.standard_normal((2, nb, D))
    q = RNG.standard_normal(D)
    ids, gap = hsa.block_select(q, kb, frames, nb, 6)
    assert list(ids) == [6, 7, 8, 15, 16, 17] and gap == math.inf
    ids, _ = hsa.block_select(q, kb, frames, nb, 1)
    sc = np.concatenate([kb[0] @ q, kb[1] @ q])
    g = [6, 7, 8, 15, 16, 17][int(np.argmax(sc))]
    assert list(ids) == [g]


def test_frame_select_takes_all_when_few():
    ft, gap = hsa.frame_select(np.ones(4), np.zeros((3, 4)), np.array([0, 1, 2]), 5)
    assert list(ft) == [0, 1, 2] and gap == math.inf


def _c1_path(wl, t_shift=0, store="bf16", dense=None, topp=None):
    """Run the c1 workload's chunks 1..4 through the oracle path."""
    cache = path.FrameCache(wl.B, wl.H, wl.D, wl.T_f, wl.blk, wl.window)
    out = None
    for c in range(1, wl.chunk + 1):
        x = chunk_inputs(wl, c)
        q, k, v = (bf16_bits_to_f32(x[n]).astype(np.float64) for n in ("q", "k", "v"))
        t0 = wl.t0_of(c) + t_shift
        hist_frames = min(wl.t0_of(c), wl.window - wl.Fc)
        k_f, k_b = hsa.budget(c, hist_frames, wl.nb, dense=wl.dense if dense is None else dense,
                              k_f_max=wl.k_f_max, k_b_fixed=wl.k_b_fixed,
                              d_base=wl.d_base, d_slope=wl.d_slope, d_pivot=wl.d_pivot)
        out = path.run_chunk(cache, q, k, v, Fh=wl.Fh, Fw=wl.Fw, Fc=wl.Fc, t0=t0,
                             k_f=k_f, k_b=k_b, dense=wl.dense if dense is None else dense,
                             store=store, topp=topp)
    return cache, out


def test_c1_sparse_selection_is_brute_force_top4():
    # Tiny case, sparse: top-4 of 9 frames, then top-4 of their 4 blocks (all).
    wl = WORKLOADS["c1s"]
    cache, out = _c1_path(wl)
    hist = out["hist"]
    assert list(hist) == list(range(9))
    for b in range(wl.B):
        for h in range(wl.H):
            for qb in range(wl.NQB):
                qbar = out["qbar_blk"][b, h, qb]
                sc = [cache.frames[t]["kf"][b, h] @ qbar for t in hist]
                want = _brute_topk(sc, 4)                     # C(9,4)=126 subsets
                assert list(out["frames"][b, h, qb]) == list(hist[want])
                assert list(out["blocks"][b, h, qb]) == list(hist[want])   # nb = 1


# --- attention ------------------------------------------------------------------

def test_attend_special_cases():
    D = 16
    k = RNG.standard_normal((10, D))
    v = RNG.standard_normal((10, D))
    q = RNG.standard_normal((3, D))
    # constant V -> that vector
    cv = np.tile(RNG.standard_normal(D), (10, 1))
    o, _ = attend(q, k, cv, 0.25)
    np.testing.assert_allclose(o, cv[:3], rtol=1e-13)
    # Q = 0 -> mean of V, lse = log(nk)
    o, lse = attend(np.zeros((2, D)), k, v, 0.25)
    np.testing.assert_allclose(o, np.tile(v.mean(0), (2, 1)), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, math.log(10), rtol=1e-14)
    # a single key -> its value
    o, _ = attend(q, k[:1], v[:1], 0.25)
    np.testing.assert_allclose(o, np.tile(v[0], (3, 1)), rtol=1e-14)
    # permutation of the keys changes nothing
    perm = RNG.permutation(10)
    o1, l1 = attend(q, k, v, 0.25)
    o2, l2 = attend(q, k[perm], v[perm], 0.25)
    np.testing.assert_allclose(o1, o2, rtol=1e-12)
    # library softmax / logsumexp
    s = 0.25 * q @ k.T
    np.testing.assert_allclose(o1, scipy.special.softmax(s, axis=1) @ v, rtol=1e-12)
    np.testing.assert_allclose(l1, scipy.special.logsumexp(s, axis=1), rtol=1e-13)


def test_full_budget_sparse_equals_dense_bruteforce():
    # c1: sparse path at full budget (k_f = 9, k_b = 9) == softmax over the
    # whole cache, computed by scipy for every query separately.
    wl = WORKLOADS["c1s"].replace(k_f_max=9, k_b_fixed=9)
    cache, out = _c1_path(wl)
    assert out["blocks"].shape[-1] == 9
    all_t = sorted(cache.frames)
    scale = 1 / math.sqrt(wl.D)
    for b in range(wl.B):
        for h in range(wl.H):
            K = np.concatenate([cache.frames[t]["k"][b, h] for t in all_t])
            V = np.concatenate([cache.frames[t]["v"][b, h] for t in all_t])
            assert K.shape[0] == 12 * 64
            for n in range(0, wl.Lq, 7):
                p = scipy.special.softmax(scale * K @ out["q_rot"][b, n, h])
                np.testing.assert_allclose(out["o"][b, n, h], p @ V, rtol=1e-10, atol=1e-12)
    # and the dense path gives the same numbers
    _, outd = _c1_path(WORKLOADS["c1"])
    np.testing.assert_allclose(outd["o"], out["o"], rtol=1e-12, atol=1e-13)


def test_global_shift_leaves_outputs_unchanged():
    # t0 = 9 and t0 = 109 (history shifted along): identical scores and outputs.
    for key in ("c1", "c1s"):
        wl = WORKLOADS[key]
        _, a = _c1_path(wl, 0, store="f64")
        _, b = _c1_path(wl, 100, store="f64")
        np.testing.assert_allclose(a["o"], b["o"], rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(a["lse"], b["lse"], rtol=1e-11)
        if a["blocks"] is not None:
            np.testing.assert_array_equal(a["blocks"] % wl.nb, b["blocks"] % wl.nb)
            np.testing.assert_array_equal(a["frames"] + 100, b["frames"])
        # the rotated tensors themselves do change with t
        assert not np.allclose(a["q_rot"], b["q_rot"])


def test_unselected_blocks_do_not_matter():
    wl = WORKLOADS["c1s"]
    cache, out = _c1_path(wl)
    b, h, qb = 0, 1, 2
    chosen = set(int(g) for g in out["blocks"][b, h, qb])
    other = [t for t in out["hist"] if t not in chosen][0]
    rows = np.arange(qb * 64, qb * 64 + 64)
    o1, _ = path.attend_chunk(out["q_rot"], cache, wl.t0, wl.Fc, out["blocks"], rows)
    cache.frames[other]["v"][b, h] += 100.0
    o2, _ = path.attend_chunk(out["q_rot"], cache, wl.t0, wl.Fc, out["blocks"], rows)
    np.testing.assert_array_equal(o1[b, rows, h], o2[b, rows, h])
    cache.frames[min(chosen)]["v"][b, h] += 100.0
    o3, _ = path.attend_chunk(out["q_rot"], cache, wl.t0, wl.Fc, out["blocks"], rows)
    assert not np.allclose(o1[b, rows, h], o3[b, rows, h])


def test_rolling_window_evicts_and_history_range():
    c = path.FrameCache(1, 1, 4, 2, 2, window=5)
    for t0 in (0, 2, 4):
        c.append(np.zeros((1, 4, 1, 4)), np.zeros((1, 4, 1, 4)), t0, 2)
    assert sorted(c.frames) == [1, 2, 3, 4, 5]
    assert list(c.history(4, 2)) == [1, 2, 3]


# --- chunk budget ------------------------------------------------------------------

def _b(wl, chunk, hist):
    return hsa.budget(chunk, hist, wl.nb, dense=wl.dense, k_f_max=wl.k_f_max,
                      d_base=wl.d_base, d_slope=wl.d_slope, d_pivot=wl.d_pivot,
                      k_b_fixed=wl.k_b_fixed)


def test_cag_literal_schedule_integers():
    # s_i = 3/4 - (i-6)/60 -> density (9+i)/60 of 3(i-1)*25 history blocks,
    # rounded half up: 11/60*75=13.75->14, 12/60*150=30, 13/60*225=48.75->49,
    # 14/60*300=70, 15/60*375=93.75->94, 16/60*450=120.
    wl = WORKLOADS["c3"]
    got = [_b(wl, i, 3 * (i - 1)) for i in range(1, 8)]
    assert got == [(0, 0), (3, 14), (6, 30), (8, 49), (8, 70), (8, 94), (8, 120)]
    assert hsa.density(wl.d_base, wl.d_slope, wl.d_pivot, 7) == Fraction(16, 60)


def test_cag_mirrored_schedule_integers():
    # density (21-i)/60: 19/60*75=23.75->24, 45, 63.75->64, 80, 93.75->94, 105
    wl = WORKLOADS["c3"].replace(d_slope=Fraction(-1, 60))
    got = [_b(wl, i, 3 * (i - 1))[1] for i in range(2, 8)]
    assert got == [24, 45, 64, 80, 94, 105]


def test_cag_other_workloads():
    assert _b(WORKLOADS["c4"], 7, 18) == (6, 104)          # 0.2*522 = 104.4
    assert _b(WORKLOADS["c5"], 80, 57) == (20, 285)        # 0.2*1425
    assert _b(WORKLOADS["c5"], 2, 3) == (3, 15)
    assert _b(WORKLOADS["c2"], 7, 18) == (18, 450)         # dense
    assert _b(WORKLOADS["c1s"], 4, 9) == (4, 4)


# ---- QKV projection + Causal-RoPE (section 2C operator fusion) ----------------

def test_qkv_identity_weight_selects_q_k_v_slices():
    # C = 3HD and W = I: q, k, v are consecutive H*D slices of x, head-major
    # inside each; q and k then rotate exactly like the pinned rope_chunk.
    from oracle import qkv
    rng = np.random.default_rng(5)
    H, D, Fh, Fw, Fc, t0 = 2, 6, 2, 3, 2, 4
    Lq = Fc * Fh * Fw
    x = rng.standard_normal((1, Lq, 3 * H * D))
    q, k, v = qkv.project(x, np.eye(3 * H * D), H, D)
    np.testing.assert_array_equal(q, x[:, :, :H * D].reshape(1, Lq, H, D))
    np.testing.assert_array_equal(k, x[:, :, H * D:2 * H * D].reshape(1, Lq, H, D))
    np.testing.assert_array_equal(v, x[:, :, 2 * H * D:].reshape(1, Lq, H, D))
    qr, kr, vv = qkv.qkv_rope(x, np.eye(3 * H * D), H, D, Fh, Fw, Fc, t0)
    np.testing.assert_allclose(qr, rope.rope_chunk(q, Fh, Fw, Fc, t0), rtol=0, atol=1e-14)
    np.testing.assert_allclose(kr, rope.rope_chunk(k, Fh, Fw, Fc, t0), rtol=0, atol=1e-14)
    np.testing.assert_array_equal(vv, v)


def test_qkv_projection_brute_force():
    # y[b, n, o] = sum_c x[b, n, c] * W[o, c], written out with loops
    from oracle import qkv
    rng = np.random.default_rng(6)
    B, Lq, C, H, D = 2, 3, 5, 1, 2
    x = rng.standard_normal((B, Lq, C))
    w = rng.standard_normal((3 * H * D, C))
    q, k, v = qkv.project(x, w, H, D)
    y = np.stack([q, k, v], axis=2).reshape(B, Lq, 3 * H * D)
    for b in range(B):
        for n in range(Lq):
            for o in range(3 * H * D):
                s = 0.0
                for c in range(C):
                    s += x[b, n, c] * w[o, c]
                assert abs(y[b, n, o] - s) < 1e-12


def test_qkv_rotation_after_projection_keeps_pair_norms_of_the_projection():
    # rotation is applied to the projected q (not to x): pair norms of q_rot
    # equal those of x W_q^T, and v is untouched by any rotation
    from oracle import qkv
    rng = np.random.default_rng(7)
    H, D, Fh, Fw, Fc, t0 = 2, 8, 2, 2, 3, 9
    x = rng.standard_normal((1, Fc * Fh * Fw, 16))
    w = rng.standard_normal((3 * H * D, 16))
    q, k, v = qkv.project(x, w, H, D)
    qr, kr, vv = qkv.qkv_rope(x, w, H, D, Fh, Fw, Fc, t0)
    n = lambda a: a[..., 0::2] ** 2 + a[..., 1::2] ** 2
    np.testing.assert_allclose(n(qr), n(q), rtol=1e-12)
    np.testing.assert_allclose(n(kr), n(k), rtol=1e-12)
    np.testing.assert_array_equal(vv, v)
    assert not np.allclose(qr, q)


# ---- CAG from the noise level ---------------------------------------------------------

def test_noise_schedule_equal_targets_give_the_base_density():
    # s_target = s_base: beta = 0, every chunk at density 1 - s_base
    d = hsa.noise_densities(10, 3, 21, 25, 0.75, 0.75)
    assert all(abs(v - 0.25) < 1e-12 for v in d.values())


def test_noise_schedule_meets_the_flop_target_and_decreases():
    # unclamped: sum d_i N_i = (1 - s_target) sum N_i; alpha_i = i^-1/2 makes
    # later chunks sparser; the closed form beta = (s_base - s_target) sum N / sum alpha N
    n, Fc, W, nb, sb, st = 12, 3, 21, 25, 0.9, 0.8
    d = hsa.noise_densities(n, Fc, W, nb, sb, st)
    N = {i: min(Fc * (i - 1), W - Fc) * nb for i in d}
    tot = sum(d[i] * N[i] for i in d)
    assert abs(tot - (1 - st) * sum(N.values())) < 1e-9 * sum(N.values())
    vals = [d[i] for i in sorted(d)]
    assert all(a > b for a, b in zip(vals, vals[1:]))
    beta = (sb - st) * sum(N.values()) / sum(N[i] / math.sqrt(i) for i in N)
    for i in d:
        assert abs(d[i] - ((1 - sb) + beta / math.sqrt(i))) < 1e-9


def test_noise_schedule_clamps_at_full_density():
    # a target denser than the base can give pushes early chunks to density 1
    d = hsa.noise_densities(6, 3, 60, 25, 0.5, 0.05)
    assert max(d.values()) == 1.0 and min(d.values()) < 1.0
    N = {i: min(3 * (i - 1), 57) * 25 for i in d}
    assert abs(sum(d[i] * N[i] for i in d) - 0.95 * sum(N.values())) < 1e-6 * sum(N.values())


def test_noise_budget_rounding_and_cap():
    assert hsa.noise_budget(1, 0, 25, 8, 0.3) == (0, 0)
    assert hsa.noise_budget(3, 6, 25, 8, 0.3) == (6, 45)        # 0.3 * 150 = 45
    assert hsa.noise_budget(3, 6, 25, 2, 0.9) == (2, 50)        # capped at 2 * 25
    assert hsa.noise_budget(2, 3, 25, 8, 0.19) == (3, 14)       # 14.25 -> 14


def test_noise_schedule_sparser_target_makes_early_chunks_sparser_first():
    # a target sparser than the base: beta < 0, early chunks lose the most
    d = hsa.noise_densities(8, 3, 21, 25, 0.7, 0.8)
    vals = [d[i] for i in sorted(d)]
    assert all(a < b for a, b in zip(vals, vals[1:]))


# ---- top-p block budget (SVG2 centroid top-p) ----------------------------------------

def _topp_inputs(seed, F=3, nb=4, D=8):
    rng = np.random.default_rng(seed)
    return rng.standard_normal(D), rng.standard_normal((F, nb, D)), np.array([2, 5, 7, 9][:F])


def test_topp_full_threshold_takes_everything_up_to_the_cap():
    q, kb, ft = _topp_inputs(1)
    ids, _ = hsa.block_select_topp(q, kb, ft, 4, 16, 5, 1.0 + 1e-12, 12)
    assert len(ids) == 12
    ids, _ = hsa.block_select_topp(q, kb, ft, 4, 16, 5, 1.0 + 1e-12, 5)
    want, _ = hsa.block_select(q, kb, ft, 4, 5)                 # the cap is a top-k
    np.testing.assert_array_equal(ids, want)


def test_topp_tiny_threshold_takes_the_top_block():
    q, kb, ft = _topp_inputs(2)
    ids, _ = hsa.block_select_topp(q, kb, ft, 4, 16, 5, 1e-9, 12)
    want, _ = hsa.block_select(q, kb, ft, 4, 1)
    np.testing.assert_array_equal(ids, want)


def test_topp_equal_scores_and_sizes_take_ceil_p_c():
    # equal masses: the prefix before candidate r holds r/C of the mass
    D, F, nb = 4, 2, 5
    q = np.zeros(D)
    kb = np.ones((F, nb, D))
    ft = np.array([0, 1])
    for p in (0.1, 0.25, 0.5, 0.61, 0.9):
        ids, _ = hsa.block_select_topp(q, kb, ft, nb, nb * 8, 8, p, F * nb)
        assert len(ids) == math.ceil(p * F * nb - 1e-12), (p, len(ids))
        np.testing.assert_array_equal(ids, np.arange(len(ids)))   # ties: lower positions


def test_topp_brute_force_shortest_prefix():
    # the chosen set is the shortest prefix of the ranking whose size-weighted
    # softmax mass reaches p (brute force over prefix lengths, written out)
    for seed in range(20):
        q, kb, ft = _topp_inputs(100 + seed, F=2, nb=3, D=6)
        T_f, blk, nb = 11, 4, 3                                     # tail block of 3 tokens
        s = kb.reshape(-1, 6) @ q
        n = np.array([4, 4, 3, 4, 4, 3], dtype=float)
        w = n * np.exp(s / math.sqrt(6))
        order = sorted(range(6), key=lambda c: (-s[c], c))
        p = 0.3 + 0.05 * (seed % 10)
        best = None
        for L in range(1, 7):
            if sum(w[c] for c in order[:L]) >= p * w.sum():
                best = L
                break
        ids, _ = hsa.block_select_topp(q, kb, ft, nb, T_f, blk, p, 6)
        want = np.sort(np.array([ft[c // 3] * 3 + c % 3 for c in order[:best]]))
        np.testing.assert_array_equal(ids, want)


def test_topp_path_full_threshold_equals_dense():
    # p just above 1 with the cap at every candidate keeps every history block
    wl = WORKLOADS["c1s"].replace(k_f_max=9, k_b_fixed=9)
    _, out = _c1_path(wl, topp=1.0 + 1e-9)
    assert np.all(out["blocks"] >= 0)
    _, outd = _c1_path(WORKLOADS["c1"])
    np.testing.assert_allclose(outd["o"], out["o"], rtol=1e-12, atol=1e-13)


def test_topp_path_rows_are_top_k_of_their_own_count():
    # a top-p row with r blocks is the top-r of the candidates, -1 after them
    wl = WORKLOADS["c1s"].replace(k_f_max=6, k_b_fixed=6)
    cache, out = _c1_path(wl, topp=0.5)
    cap = out["blocks"].shape[-1]
    counts = (out["blocks"] >= 0).sum(-1)
    assert counts.min() >= 1 and counts.max() <= cap and counts.min() < cap
    for b in range(wl.B):
        for h in range(wl.H):
            for qb in range(wl.NQB):
                row = out["blocks"][b, h, qb]
                r = counts[b, h, qb]
                assert np.all(row[r:] == -1)
                ft = out["frames"][b, h, qb]
                kb = np.stack([cache.frames[t]["kb"][b, h] for t in ft])
                want, _ = hsa.block_select(out["qbar_blk"][b, h, qb], kb, ft, wl.nb, r)
                np.testing.assert_array_equal(row[:r], want)


def test_denoising_passes_leave_no_trace():
    # every pass of a chunk writes that chunk's frames; only the last (clean)
    # pass is seen by later chunks, and a pass evicts nothing inside the
    # chunk's own history
    wl = WORKLOADS["r64s"].with_chunk(4)
    def run(noisy_passes):
        cache = path.FrameCache(wl.B, wl.H, wl.D, wl.T_f, wl.blk, wl.window)
        outs = {}
        for c in range(1, 5):
            t0 = wl.t0_of(c)
            hist_frames = min(t0, wl.window - wl.Fc)
            k_f, k_b = hsa.budget(c, hist_frames, wl.nb, dense=False, k_f_max=wl.k_f_max,
                                  d_base=wl.d_base, d_slope=wl.d_slope, d_pivot=wl.d_pivot)
            passes = [chunk_inputs(wl, c, layer=7 + i) for i in range(noisy_passes if c == 2 else 0)]
            passes.append(chunk_inputs(wl, c))
            for x in passes:
                q, k, v = (bf16_bits_to_f32(x[n]).astype(np.float64) for n in ("q", "k", "v"))
                outs[c] = path.run_chunk(cache, q, k, v, Fh=wl.Fh, Fw=wl.Fw, Fc=wl.Fc, t0=t0,
                                         k_f=k_f, k_b=k_b, dense=False)
        return outs
    a, b = run(0), run(2)
    for c in (2, 3, 4):
        np.testing.assert_array_equal(a[c]["o"], b[c]["o"])


# --- attention on ragged frames (several blocks per frame, a short tail) -----------
#
# Frames of 5 x 9 = 45 tokens over 16-token blocks: blocks [0, 16), [16, 32) and
# the 13-token tail [32, 45). Two history frames (t = 0, 1) and a chunk of two
# frames (t = 2, 3) whose 90 queries form six query blocks. The rows of each
# query block and the token range of each picked block are written out by hand
# below (not derived from the block size), so a slip in the oracle's row -> query
# block map or in its tail slicing changes some key set and fails the test.

_RAG_D, _RAG_TF, _RAG_BLK = 16, 45, 16
# query block -> rows of the chunk (frame 2 holds rows 0..44, frame 3 rows 45..89)
_RAG_QROWS = {0: range(0, 16), 1: range(16, 32), 2: range(32, 45),
              3: range(45, 61), 4: range(61, 77), 5: range(77, 90)}
# block id t*3 + j -> (frame t, first token, end token) of the picked history block
_RAG_BLOCKS = {0: (0, 0, 16), 1: (0, 16, 32), 2: (0, 32, 45),
               3: (1, 0, 16), 4: (1, 16, 32), 5: (1, 32, 45)}
# picks per query block (ascending ids, as the selection reports them)
_RAG_PICKS = {0: [2], 1: [1, 3], 2: [2, 5], 3: [0, 4], 4: [3, 4, 5], 5: [1]}


def _ragged_case():
    rng = np.random.default_rng(4242)
    D, T_f = _RAG_D, _RAG_TF
    hist_k = rng.standard_normal((1, 2 * T_f, 1, D))
    hist_v = rng.standard_normal((1, 2 * T_f, 1, D))
    cur_k = rng.standard_normal((1, 2 * T_f, 1, D))
    cur_v = rng.standard_normal((1, 2 * T_f, 1, D))
    q = rng.standard_normal((1, 2 * T_f, 1, D))
    cache = path.FrameCache(1, 1, D, T_f, _RAG_BLK, window=8)
    cache.append(hist_k, hist_v, 0, 2)
    cache.append(cur_k, cur_v, 2, 2)
    blocks = np.zeros((1, 1, 6, 3), dtype=np.int64) - 1
    for qb, ids in _RAG_PICKS.items():
        blocks[0, 0, qb, :len(ids)] = ids
    return cache, q, blocks, (hist_k, hist_v, cur_k, cur_v)


def _ragged_keys_by_hand(qb, raw):
    hist_k, hist_v, cur_k, cur_v = raw
    ks, vs = [], []
    for g in _RAG_PICKS[qb]:
        t, lo, hi = _RAG_BLOCKS[g]
        ks.append(hist_k[0, t * _RAG_TF + lo:t * _RAG_TF + hi, 0])
        vs.append(hist_v[0, t * _RAG_TF + lo:t * _RAG_TF + hi, 0])
    ks.append(cur_k[0, :, 0])                  # the whole current chunk
    vs.append(cur_v[0, :, 0])
    return np.concatenate(ks), np.concatenate(vs)


def test_ragged_frames_key_sets_match_hand_built_ranges():
    cache, q, blocks, raw = _ragged_case()
    for qb in range(6):
        k, v = path.keys_of_query_block(cache, 0, 0, 2, 2, blocks[0, 0, qb])
        kw, vw = _ragged_keys_by_hand(qb, raw)
        np.testing.assert_array_equal(k, kw)
        np.testing.assert_array_equal(v, vw)
    # the tail blocks hold 13 tokens, the others 16
    k2, _ = path.keys_of_query_block(cache, 0, 0, 2, 2, np.array([2]))
    assert k2.shape[0] == 13 + 90


def test_ragged_frames_attention_brute_force():
    cache, q, blocks, raw = _ragged_case()
    o, lse = path.attend_chunk(q, cache, 2, 2, blocks)
    scale = 1 / math.sqrt(_RAG_D)
    seen = set()
    for qb, rows in _RAG_QROWS.items():
        K, V = _ragged_keys_by_hand(qb, raw)
        for r in rows:
            s = scale * K @ q[0, r, 0]
            np.testing.assert_allclose(o[0, r, 0], scipy.special.softmax(s) @ V, rtol=1e-11, atol=1e-13)
            np.testing.assert_allclose(lse[0, 0, r], scipy.special.logsumexp(s), rtol=1e-13)
            seen.add(r)
    assert seen == set(range(90))
    # a row subset gives the same numbers for those rows
    rows = np.array([0, 31, 32, 44, 45, 60, 61, 89])
    o2, _ = path.attend_chunk(q, cache, 2, 2, blocks, rows)
    np.testing.assert_allclose(o2[0, rows], o[0, rows], rtol=1e-13, atol=1e-15)
