"""Host-side checks of the C ABI (no GPU needed).

The library must load, export every function ``include/cva.h`` declares,
and validate arguments on the host before it would launch anything. Its
host-only computations (rotary tables, chunk budget, cache and workspace
sizes, history range) are checked against the oracle or closed forms.
"""
import ctypes
import os
import re
from fractions import Fraction

import numpy as np
import pytest

from cva_workload import WORKLOADS
from oracle import hsa as o_hsa
from oracle import rope as o_rope

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ops():
    from autoregressive_video_dit_b200 import ops as _ops
    return _ops


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "cva.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(cva_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol(ops):
    names = _declared_functions()
    assert len(names) >= 15
    lib = ctypes.CDLL(ops._LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert set(names) == set(ops.EXPORTED)


def test_version_and_last_error(ops):
    assert ops.lib.cva_version() == 1
    assert isinstance(ops.last_error(), str)


@pytest.mark.parametrize("D", [64, 128])
def test_rope_tables_match_oracle(ops, D):
    t = ops.rope3d_precompute(D, 240, 45, 80)
    ref = o_rope.tables(D, 240, 45, 80)
    for (name_c, name_s), (c, s) in zip((("cos_t", "sin_t"), ("cos_h", "sin_h"), ("cos_w", "sin_w")), ref):
        np.testing.assert_allclose(t[name_c], c, rtol=0, atol=6e-8)
        np.testing.assert_allclose(t[name_s], s, rtol=0, atol=6e-8)
    assert ops.rope_axis_pairs(D) == o_rope.axis_split(D)


@pytest.mark.parametrize("D", [64, 128])
def test_position_table_repeats_the_axis_tables(ops, D):
    # the per-position expansion holds exactly the per-axis floats, (1, 0) for
    # the temporal pairs, and its pairs rotate like the oracle's angles
    Fh, Fw = 7, 11
    t = ops.rope3d_precompute(D, 8, Fh, Fw)
    tok = t["cs_tok"]
    pt, ph, pw = ops.rope_axis_pairs(D)
    assert tok.shape == (Fh, Fw, D // 2, 2)
    np.testing.assert_array_equal(tok[:, :, :pt, 0], 1.0)
    np.testing.assert_array_equal(tok[:, :, :pt, 1], 0.0)
    for h in range(Fh):
        for w in range(Fw):
            np.testing.assert_array_equal(tok[h, w, pt:pt + ph, 0], t["cos_h"][h])
            np.testing.assert_array_equal(tok[h, w, pt:pt + ph, 1], t["sin_h"][h])
            np.testing.assert_array_equal(tok[h, w, pt + ph:, 0], t["cos_w"][w])
            np.testing.assert_array_equal(tok[h, w, pt + ph:, 1], t["sin_w"][w])
    ang = o_rope.pair_angles(D, np.zeros(Fh * Fw), np.repeat(np.arange(Fh), Fw), np.tile(np.arange(Fw), Fh))
    np.testing.assert_allclose(tok[..., 0].reshape(Fh * Fw, -1), np.cos(ang), rtol=0, atol=6e-8)
    np.testing.assert_allclose(tok[..., 1].reshape(Fh * Fw, -1), np.sin(ang), rtol=0, atol=6e-8)


def test_copy_rows_2d_validates_before_launching(ops):
    fake = ctypes.c_void_p(1 << 41)
    f = ops.lib.cva_copy_rows_2d
    assert f(fake, fake, 0, 4, 16, 16, 16, 16, 16, None) == 0           # nothing to copy
    assert f(fake, fake, 2, 2, 24, 48, 24, 24, 48, None) == ops.CVA_EINVAL  # 24-byte rows
    assert f(fake, fake, 2, 2, 32, 40, 32, 32, 64, None) == ops.CVA_EINVAL  # stride not 16-aligned
    assert f(ctypes.c_void_p((1 << 41) + 8), fake, 2, 2, 32, 64, 32, 32, 64, None) == ops.CVA_EINVAL
    assert f(None, fake, 2, 2, 32, 64, 32, 32, 64, None) == ops.CVA_EINVAL
    assert f(fake, fake, -1, 2, 32, 64, 32, 32, 64, None) == ops.CVA_EINVAL


def _lib_budget(ops, wl, chunk, hist):
    return ops.cag_budget(chunk, hist, wl.nb, dense=wl.dense, k_f_max=wl.k_f_max,
                          d_base=(wl.d_base.numerator, wl.d_base.denominator),
                          d_slope=(wl.d_slope.numerator, wl.d_slope.denominator),
                          pivot=wl.d_pivot, k_b_fixed=wl.k_b_fixed)


def _oracle_budget(wl, chunk, hist):
    return o_hsa.budget(chunk, hist, wl.nb, dense=wl.dense, k_f_max=wl.k_f_max, d_base=wl.d_base,
                        d_slope=wl.d_slope, d_pivot=wl.d_pivot, k_b_fixed=wl.k_b_fixed)


@pytest.mark.parametrize("key", sorted(WORKLOADS))
def test_cag_budget_matches_oracle(ops, key):
    wl = WORKLOADS[key]
    for chunk in range(1, 90):
        hist = min(wl.Fc * (chunk - 1), wl.window - wl.Fc)
        assert _lib_budget(ops, wl, chunk, hist) == _oracle_budget(wl, chunk, hist), (key, chunk)


def test_cag_budget_mirrored_and_extreme_slopes(ops):
    wl = WORKLOADS["c3"]
    for slope in (Fraction(-1, 60), Fraction(1, 3), Fraction(-1, 2), Fraction(7, 13)):
        w2 = wl.replace(d_slope=slope)
        for chunk in range(1, 12):
            hist = 3 * (chunk - 1)
            assert _lib_budget(ops, w2, chunk, hist) == _oracle_budget(w2, chunk, hist)


def test_shape_validation(ops):
    s = ops.make_shape(1, 2, 96, 4, 4, 3, 64)
    n = ctypes.c_size_t()
    assert ops.lib.cva_kv_cache_bytes(ctypes.byref(s), 6, ctypes.byref(n)) == ops.CVA_ENOTSUP
    s = ops.make_shape(1, 2, 128, 4, 4, 3, 32)
    assert ops.lib.cva_kv_cache_bytes(ctypes.byref(s), 6, ctypes.byref(n)) == ops.CVA_ENOTSUP
    s = ops.make_shape(0, 2, 128, 4, 4, 3, 64)
    assert ops.lib.cva_kv_cache_bytes(ctypes.byref(s), 6, ctypes.byref(n)) == ops.CVA_EINVAL
    s = ops.make_shape(1, 2, 128, 4, 4, 3, 64)
    assert ops.lib.cva_kv_cache_bytes(ctypes.byref(s), 2, ctypes.byref(n)) == ops.CVA_EINVAL
    assert ops.lib.cva_kv_cache_bytes(None, 6, ctypes.byref(n)) == ops.CVA_EINVAL
    assert "head_dim" in ops.last_error() or "shape" in ops.last_error()


def _fake_cache(ops, shape, window, t_begin=0):
    c = ops.KVCache()
    nbytes = ops.kv_cache_bytes(shape, window)
    rc = ops.lib.cva_kv_cache_init(ctypes.byref(c), ctypes.c_void_p(1 << 40), nbytes,
                                   ctypes.byref(shape), window, t_begin)
    assert rc == ops.CVA_OK, ops.last_error()
    return c, nbytes


def test_cache_layout_sizes(ops):
    wl = WORKLOADS["c2"]
    s = ops.make_shape(wl.B, wl.H, wl.D, wl.Fh, wl.Fw, wl.Fc, wl.blk)
    c, nbytes = _fake_cache(ops, s, wl.window)
    kv = wl.B * wl.H * wl.window * wl.T_pad * wl.D * 2
    assert c.v - c.k == kv and c.kpool_blk - c.v == kv
    assert c.kpool_frm - c.kpool_blk == wl.B * wl.H * wl.window * wl.nb * wl.D * 4
    assert nbytes == 2 * kv + wl.B * wl.H * wl.window * (wl.nb + 1) * wl.D * 4
    small = ops.KVCache()
    assert ops.lib.cva_kv_cache_init(ctypes.byref(small), ctypes.c_void_p(1 << 40), nbytes - 1,
                                     ctypes.byref(s), wl.window, 0) == ops.CVA_ENOMEM
    assert ops.lib.cva_kv_cache_init(ctypes.byref(small), ctypes.c_void_p((1 << 40) + 16), nbytes,
                                     ctypes.byref(s), wl.window, 0) == ops.CVA_EINVAL


def test_history_frames_range(ops):
    s = ops.make_shape(1, 1, 64, 4, 4, 3, 64)
    c, _ = _fake_cache(ops, s, 60)
    lo, n = ctypes.c_int32(), ctypes.c_int32()
    for t0, want in ((0, (0, 0)), (3, (0, 3)), (57, (0, 57)), (60, (3, 57)), (237, (180, 57))):
        assert ops.lib.cva_history_frames(ctypes.byref(c), t0, ctypes.byref(lo), ctypes.byref(n)) == 0
        assert (lo.value, n.value) == want
    c2, _ = _fake_cache(ops, s, 12, t_begin=100)
    assert ops.lib.cva_history_frames(ctypes.byref(c2), 109, ctypes.byref(lo), ctypes.byref(n)) == 0
    assert (lo.value, n.value) == (100, 9)
    assert ops.lib.cva_history_frames(ctypes.byref(c2), 99, ctypes.byref(lo), ctypes.byref(n)) == ops.CVA_ERANGE


def test_select_rejects_budget_beyond_candidates(ops):
    wl = WORKLOADS["r64"]
    s = ops.make_shape(wl.B, wl.H, wl.D, wl.Fh, wl.Fw, wl.Fc, wl.blk)
    c, _ = _fake_cache(ops, s, wl.window)
    fake = ctypes.c_void_p(1 << 41)
    # t0 = 6: 6 history frames, k_f = 4 -> 8 candidate blocks
    rc = ops.lib.cva_hsa_select(fake, ctypes.byref(c), 6, 4, 9, None, fake, fake, None)
    assert rc == ops.CVA_ERANGE and "k_b" in ops.last_error()
    rc = ops.lib.cva_hsa_select(fake, ctypes.byref(c), 6, 0, 0, None, fake, fake, None)
    assert rc == ops.CVA_ERANGE
    rc = ops.lib.cva_hsa_select(None, ctypes.byref(c), 6, 4, 4, None, fake, fake, None)
    assert rc == ops.CVA_EINVAL


def test_select_topp_rejects_bad_threshold_and_cap(ops):
    wl = WORKLOADS["r64"]
    s = ops.make_shape(wl.B, wl.H, wl.D, wl.Fh, wl.Fw, wl.Fc, wl.blk)
    c, _ = _fake_cache(ops, s, wl.window)
    fake = ctypes.c_void_p(1 << 41)
    f = ops.lib.cva_hsa_select_topp
    for p in (0.0, -0.5, 1.5, float("nan")):
        assert f(fake, ctypes.byref(c), 6, 4, 8, p, None, fake, fake, None) == ops.CVA_ERANGE
        assert "p must" in ops.last_error()
    assert f(fake, ctypes.byref(c), 6, 4, 0, 0.5, None, fake, fake, None) == ops.CVA_ERANGE
    assert f(fake, ctypes.byref(c), 6, 4, 9, 0.5, None, fake, fake, None) == ops.CVA_ERANGE   # 9 > 8 candidates
    assert f(None, ctypes.byref(c), 6, 4, 8, 0.5, None, fake, fake, None) == ops.CVA_EINVAL
    g = ops.lib.cva_chunk_attention_topp
    assert g(fake, fake, fake, ctypes.byref(c), None, 6, 4, 8, 0.0, fake, 1 << 30, fake, None,
             None) == ops.CVA_ERANGE
    assert g(fake, fake, fake, ctypes.byref(c), None, 6, 0, 8, 0.5, fake, 1 << 30, fake, None,
             None) == ops.CVA_ERANGE


def test_attention_rejects_oversized_key_lists(ops):
    # 256 history frames x 25 blocks exceed the per-tile key-unit list
    s = ops.make_shape(1, 1, 128, 30, 52, 3, 64)
    c, _ = _fake_cache(ops, s, 259)
    fake = ctypes.c_void_p(1 << 41)
    rc = ops.lib.cva_blocksparse_attn_fwd(fake, ctypes.byref(c), 256, None, None, 0, fake, None,
                                          None, 0, None)
    assert rc == ops.CVA_ENOTSUP


def test_workspace_bytes(ops):
    wl = WORKLOADS["c3"]
    s = ops.make_shape(wl.B, wl.H, wl.D, wl.Fh, wl.Fw, wl.Fc, wl.blk)
    r = lambda x: (x + 255) // 256 * 256
    bhq = wl.B * wl.H * wl.NQB
    # attention scratch: partial O, max and sum of up to 160 key-range pieces
    attn = r(160 * 128 * wl.D * 4) + r(160 * 128 * 2 * 4)
    MT = -(-wl.Fc * wl.T_pad // 128)   # 128-row query tiles per head; a pair of query blocks each
    want = (r(wl.B * wl.H * wl.Fc * wl.T_pad * wl.D * 2) + r(bhq * wl.D * 4) + r(bhq * 8 * 4)
            + r(bhq * 120 * 4) + r(bhq * 4) + r(wl.B * wl.H * MT * 2 * 4) + attn)
    assert ops.chunk_workspace_bytes(s, 8, 120) == want
    assert ops.attn_workspace_bytes(s, 120) == attn


@pytest.mark.parametrize("n,Fc,W,nb,sb,st", [(10, 3, 21, 25, 0.75, 0.7), (80, 3, 60, 25, 0.9, 0.8),
                                              (7, 3, 21, 29, 0.8, 0.8), (6, 3, 60, 25, 0.5, 0.05),
                                              (8, 3, 21, 25, 0.7, 0.8), (30, 2, 9, 3, 1.0, 0.6)])
def test_noise_schedule_matches_oracle(ops, n, Fc, W, nb, sb, st):
    want = o_hsa.noise_densities(n, Fc, W, nb, sb, st)
    got = ops.cag_noise_densities(n, Fc, W, nb, sb, st)
    assert got.keys() == want.keys()
    for i in want:
        assert got[i] == want[i], (i, got[i], want[i])     # same fp64 steps, same values
        hist = min(Fc * (i - 1), W - Fc)
        assert ops.cag_density_budget(i, hist, nb, 8, got[i]) == o_hsa.noise_budget(i, hist, nb, 8, want[i])


def test_noise_schedule_rejects_bad_arguments(ops):
    with pytest.raises(ops.CvaError):
        ops.cag_noise_densities(1, 3, 21, 25, 0.75, 0.7)
    with pytest.raises(ops.CvaError):
        ops.cag_noise_densities(5, 3, 2, 25, 0.75, 0.7)
    with pytest.raises(ops.CvaError):
        ops.cag_noise_densities(5, 3, 21, 25, 1.5, 0.7)
