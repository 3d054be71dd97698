"""GPU parity: every step of the CUDA path against the fp64 oracle.

Staged tests feed each kernel the oracle's own (bfloat16-rounded) inputs
for that step, so a mismatch points at one kernel. End-to-end tests run the
fused chunk call from raw seeded inputs over a whole sequence of chunks.
Tolerances: RoPE 1e-2 absolute (or the bf16 rounding bound of the value);
pooled means 1e-5 relative to the row scale; selection identical except
where the oracle's boundary gap is below 1e-5 relative; attention max-abs
2e-2 and mean-abs 2e-3.
"""
import math

import numpy as np
import pytest

from cva_workload import WORKLOADS, key_centres
from oracle import hsa as o_hsa
from oracle import path as o_path
from oracle import rope as o_rope

from _util import (MAX_ABS, MEAN_ABS, attn_errors, bits_to_f64, f64_to_bits, from_dev, inputs,
                   lib_budget, oracle_budget, hist_count, rope_tol, sample_rows, check_selection, ws_lists, oracle_run,
                   shape_of, to_dev, mutual_best_pairs)

pytestmark = pytest.mark.gpu

SMALL = ["c1", "c1s", "r64", "r128", "r64s"]
SMALL_SPARSE = ["c1s", "r64", "r128", "r64s"]


@pytest.fixture(scope="module")
def ops():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from autoregressive_video_dit_b200 import ops as _ops
    _ops.device_status(clear=True)
    return _ops


def _tables(ops, wl, t_begin=0):
    max_t = t_begin + wl.Fc * max(wl.chunk, wl.chunks) + wl.Fc
    return ops.DeviceRopeTables(wl.D, max_t, wl.Fh, wl.Fw)


def _sub(wl, heads):
    return wl if heads is None else wl.replace(H=len(heads))


_oracle_run = oracle_run


def _head_major(wl, q_rot_tok):
    """[B, Lq, H, D] -> [B, H, Fc*T_pad, D] with zero pad rows."""
    B, Lq, H, D = q_rot_tok.shape
    out = np.zeros((B, H, wl.Fc, wl.T_pad, D), dtype=q_rot_tok.dtype)
    x = np.transpose(q_rot_tok, (0, 2, 1, 3)).reshape(B, H, wl.Fc, wl.T_f, D)
    out[:, :, :, :wl.T_f] = x
    return out.reshape(B, H, wl.Fc * wl.T_pad, D)


def _gpu_cache_from_oracle(ops, wl, run, t_begin=0):
    """GPU cache holding exactly the oracle's bf16 rotated keys (append without rotation)."""
    cache = ops.DeviceKVCache(shape_of(wl), wl.window, t_begin)
    for t0, k_rot, v_bits in run["hist"]:
        ops.kv_append(to_dev(f64_to_bits(k_rot)), to_dev(v_bits), cache, None, t0)
    ops.kv_append(to_dev(f64_to_bits(run["k_rot"])), to_dev(run["x"]["v"]), cache, None, run["t0"])
    return cache


# ---- step 1: RoPE ---------------------------------------------------------------

@pytest.mark.parametrize("key", SMALL + ["c2"])
def test_rope3d_apply(ops, key):
    import torch
    wl = WORKLOADS[key]
    x = inputs(wl, wl.chunk)
    tabs = _tables(ops, wl)
    shp = shape_of(wl)
    for name in ("q", "k"):
        want = o_rope.rope_chunk(bits_to_f64(x[name]), wl.Fh, wl.Fw, wl.Fc, wl.t0)
        xd = to_dev(x[name])
        y0 = torch.empty_like(xd)
        ops.rope3d_apply(xd, y0, tabs, shp, wl.t0, 0)
        got = bits_to_f64(from_dev(y0))
        assert np.all(np.abs(got - want) <= rope_tol(want)), f"{name}: max err {np.abs(got - want).max()}"
        # exact agreement with the oracle's own bf16 rounding almost everywhere
        frac_diff = np.mean(got != o_path.round_bf16(want))
        assert frac_diff < 1e-3
        y1 = torch.full((wl.B, wl.H, wl.Fc * wl.T_pad, wl.D), float("nan"), dtype=torch.bfloat16,
                        device="cuda")
        ops.rope3d_apply(xd, y1, tabs, shp, wl.t0, 1)
        torch.cuda.synchronize()
        hm = bits_to_f64(from_dev(y1)).reshape(wl.B, wl.H, wl.Fc, wl.T_pad, wl.D)
        np.testing.assert_array_equal(hm[:, :, :, :wl.T_f],
                                      np.transpose(got, (0, 2, 1, 3)).reshape(wl.B, wl.H, wl.Fc, wl.T_f, wl.D))
        assert np.all(hm[:, :, :, wl.T_f:] == 0)


@pytest.mark.parametrize("key", ["c1", "r64", "r64s"])
def test_rope_without_the_position_table(ops, key):
    # tables without the per-position expansion take the per-pair lookup kernel:
    # same results as with it
    import torch
    wl = WORKLOADS[key]
    x = inputs(wl, wl.chunk)
    tabs = _tables(ops, wl)
    shp = shape_of(wl)
    xd = to_dev(x["q"])
    y_tok = torch.empty_like(xd)
    ops.rope3d_apply(xd, y_tok, tabs, shp, wl.t0, 0)
    tabs.struct.cs_tok = None
    y_plain = torch.empty_like(xd)
    ops.rope3d_apply(xd, y_plain, tabs, shp, wl.t0, 0)
    cache = ops.DeviceKVCache(shp, wl.window)
    ops.kv_append(to_dev(x["k"]), to_dev(x["v"]), cache, tabs, wl.t0)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(from_dev(y_plain), from_dev(y_tok))
    want = o_rope.rope_chunk(bits_to_f64(x["k"]), wl.Fh, wl.Fw, wl.Fc, wl.t0)
    kc = bits_to_f64(from_dev(cache.k))
    for f in range(wl.Fc):
        got = kc[:, :, (wl.t0 + f) % wl.window, :wl.T_f]
        w = np.transpose(want[:, f * wl.T_f:(f + 1) * wl.T_f], (0, 2, 1, 3))
        assert np.all(np.abs(got - w) <= rope_tol(w))


# ---- step 2 (+ K pooling): append ------------------------------------------------------

@pytest.mark.parametrize("key", SMALL)
def test_kv_append_rotates_copies_and_pools(ops, key):
    import torch
    wl = WORKLOADS[key]
    shp = shape_of(wl)
    tabs = _tables(ops, wl)
    cache = ops.DeviceKVCache(shp, wl.window)
    x = inputs(wl, wl.chunk)
    ops.kv_append(to_dev(x["k"]), to_dev(x["v"]), cache, tabs, wl.t0)
    torch.cuda.synchronize()
    k_want = o_rope.rope_chunk(bits_to_f64(x["k"]), wl.Fh, wl.Fw, wl.Fc, wl.t0)
    kc = bits_to_f64(from_dev(cache.k))
    vc = from_dev(cache.v)
    for f in range(wl.Fc):
        slot = (wl.t0 + f) % wl.window
        kf = kc[:, :, slot]                                     # [B,H,T_pad,D]
        want = np.transpose(k_want[:, f * wl.T_f:(f + 1) * wl.T_f], (0, 2, 1, 3))
        assert np.all(np.abs(kf[:, :, :wl.T_f] - want) <= rope_tol(want))
        assert np.all(kf[:, :, wl.T_f:] == 0)
        np.testing.assert_array_equal(vc[:, :, slot, :wl.T_f],
                                      np.transpose(x["v"][:, f * wl.T_f:(f + 1) * wl.T_f], (0, 2, 1, 3)))
        assert np.all(vc[:, :, slot, wl.T_f:] == 0)
        # pools of the stored keys
        pb = cache.kpool_blk[:, :, slot].cpu().numpy().astype(np.float64)
        pf = cache.kpool_frm[:, :, slot].cpu().numpy().astype(np.float64)
        want_b = o_hsa.block_means(kf[:, :, :wl.T_f], wl.blk)
        want_f = o_hsa.frame_mean(kf[:, :, :wl.T_f])
        np.testing.assert_allclose(pb, want_b, rtol=0, atol=2e-6 * max(1.0, np.abs(want_b).max()))
        np.testing.assert_allclose(pf, want_f, rtol=0, atol=2e-6 * max(1.0, np.abs(want_f).max()))


@pytest.mark.parametrize("key", ["r64", "r128"])
def test_kv_append_without_rotation_is_a_copy(ops, key):
    import torch
    wl = WORKLOADS[key]
    cache = ops.DeviceKVCache(shape_of(wl), wl.window)
    x = inputs(wl, 2)
    ops.kv_append(to_dev(x["k"]), to_dev(x["v"]), cache, None, wl.t0_of(2))
    torch.cuda.synchronize()
    kc = from_dev(cache.k)
    for f in range(wl.Fc):
        slot = (wl.t0_of(2) + f) % wl.window
        np.testing.assert_array_equal(kc[:, :, slot, :wl.T_f],
                                      np.transpose(x["k"][:, f * wl.T_f:(f + 1) * wl.T_f], (0, 2, 1, 3)))


# ---- step 3: query pooling --------------------------------------------------------------

@pytest.mark.parametrize("key", SMALL + ["c3"])
def test_hsa_compress(ops, key):
    import torch
    wl = WORKLOADS[key]
    heads = [0, wl.H - 1] if wl.H > 4 else None
    wl = _sub(wl, heads) if heads else wl
    x = inputs(WORKLOADS[key], wl.chunk, 0, heads)
    q_rot, _ = o_path.rotate_chunk(bits_to_f64(x["q"]), bits_to_f64(x["k"]), wl.Fh, wl.Fw, wl.Fc, wl.t0)
    want_b, want_f = o_path.pool_queries(q_rot, wl.T_f, wl.blk, wl.Fc)
    qd = to_dev(f64_to_bits(_head_major(wl, q_rot)))
    pb = torch.empty((wl.B, wl.H, wl.NQB, wl.D), dtype=torch.float32, device="cuda")
    pf = torch.empty((wl.B, wl.H, wl.Fc, wl.D), dtype=torch.float32, device="cuda")
    ops.hsa_compress(qd, shape_of(wl), pb, pf)
    torch.cuda.synchronize()
    np.testing.assert_allclose(pb.cpu().numpy(), want_b, rtol=0, atol=2e-6 * max(1, np.abs(want_b).max()))
    np.testing.assert_allclose(pf.cpu().numpy(), want_f, rtol=0, atol=2e-6 * max(1, np.abs(want_f).max()))


# ---- step 4: selection ------------------------------------------------------------------

def _staged_select(ops, wl, run, t_begin=0):
    import torch
    cache = _gpu_cache_from_oracle(ops, wl, run, t_begin)
    qd = to_dev(f64_to_bits(_head_major(wl, run["q_rot"])))
    pb = torch.empty((wl.B, wl.H, wl.NQB, wl.D), dtype=torch.float32, device="cuda")
    ops.hsa_compress(qd, shape_of(wl), pb)
    k_f, k_b = run["k_f"], run["k_b"]
    F = len(run["cache"].history(run["t0"], wl.Fc))
    kfe = min(k_f, F)
    fi = torch.full((wl.B, wl.H, wl.NQB, max(kfe, 1)), -7, dtype=torch.int32, device="cuda")
    bi = torch.full((wl.B, wl.H, wl.NQB, max(k_b, 1)), -7, dtype=torch.int32, device="cuda")
    bc = torch.full((wl.B, wl.H, wl.NQB), -7, dtype=torch.int32, device="cuda")
    ops.hsa_select(pb, cache, run["t0"], k_f, k_b, fi, bi, bc)
    torch.cuda.synchronize()
    return cache, qd, fi.cpu().numpy(), bi.cpu().numpy(), bc.cpu().numpy()


@pytest.mark.parametrize("key", SMALL_SPARSE)
def test_hsa_select_staged(ops, key):
    wl = WORKLOADS[key]
    run = _oracle_run(wl, wl.chunk)
    _, _, fi, bi, bc = _staged_select(ops, wl, run)
    n, bad, near, _ = check_selection(run, fi, bi, bc)
    assert bad == 0 and near <= 0.02 * n, (bad, near, n)
    kfe = run["frames"].shape[-1]
    ok = (run["gap_f"] >= 1e-5)
    np.testing.assert_array_equal(fi[..., :kfe][ok], run["frames"][ok])


@pytest.mark.parametrize("chunk", [2, 4, 7])
def test_hsa_select_staged_c3_full_size(ops, chunk):
    wl = WORKLOADS["c3"].with_chunk(chunk)
    heads = [0, 5, 11]
    run = _oracle_run(wl, chunk, heads)
    k_f, k_b = lib_budget(wl, chunk)
    assert (k_f, k_b) == (run["k_f"], run["k_b"])
    _, _, fi, bi, bc = _staged_select(ops, _sub(wl, heads), run)
    n, bad, near, _ = check_selection(run, fi, bi, bc)
    assert bad == 0 and near <= 0.02 * n, (bad, near, n)


def _max_history_workload(k_b):
    # 256 history frames (the selection's limit) of 16x16 tokens in 4 blocks:
    # the second level ranks 1024 candidates (its limit), k_b of them kept
    return WORKLOADS["c1s"].replace(H=1, D=64, Fh=16, Fw=16, window=259, chunk=87, k_f_max=256,
                                    k_b_fixed=k_b)


@pytest.mark.parametrize("k_b", [700, 1024])
def test_select_and_attention_at_the_size_limits(ops, k_b):
    wl = _max_history_workload(k_b)
    run = _oracle_run(wl, wl.chunk)
    assert run["k_f"] == 256 and run["k_b"] == k_b and len(run["hist"]) == 86
    assert run["frames"].shape[-1] == 256 and run["blocks"].shape[-1] == k_b
    _, _, fi, bi, bc = _staged_select(ops, wl, run)
    n, bad, near, _ = check_selection(run, fi, bi, bc)
    assert bad == 0 and near <= 0.1 * n, (bad, near, n)
    _check_attention(ops, wl, run, run["blocks"], split=True)


# ---- step 5: attention ------------------------------------------------------------------

def _check_attention(ops, wl, run, blocks, rows=None, t_begin=0, split=False):
    import torch
    cache = _gpu_cache_from_oracle(ops, wl, run, t_begin)
    ws = None
    if split:  # with the scratch the tiles of the last partial wave run as key-range pieces
        ws = torch.empty(ops.attn_workspace_bytes(cache.shape, 0), dtype=torch.uint8, device="cuda")
    qd = to_dev(f64_to_bits(_head_major(wl, run["q_rot"])))
    out = torch.full((wl.B, wl.Lq, wl.H, wl.D), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((wl.B, wl.H, wl.Lq), float("nan"), dtype=torch.float32, device="cuda")
    if blocks is None:
        ops.blocksparse_attn_fwd(qd, cache, run["t0"], None, None, 0, out, lse, ws)
    else:
        kb = blocks.shape[-1]
        # at least one element: an empty tensor has a NULL data pointer, which means "dense"
        padded = np.zeros(blocks.shape[:-1] + (max(kb, 1),), dtype=np.int32)
        padded[..., :kb] = blocks
        bi = torch.from_numpy(padded).cuda()
        bc = torch.full(blocks.shape[:-1], kb, dtype=torch.int32, device="cuda")
        ops.blocksparse_attn_fwd(qd, cache, run["t0"], bi, bc, kb, out, lse, ws)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    o_want, l_want = o_path.attend_chunk(run["q_rot"], run["cache"], run["t0"], wl.Fc, blocks, rows)
    got = bits_to_f64(from_dev(out))
    gl = lse.cpu().numpy().astype(np.float64)
    sel = np.arange(wl.Lq) if rows is None else rows
    mx, mean, rel = attn_errors(got[:, sel], o_want[:, sel])
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean, rel)
    np.testing.assert_allclose(gl[:, :, sel], l_want[:, :, sel], rtol=0, atol=2e-3)
    return mx, mean, rel


@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("key", SMALL)
def test_attention_staged(ops, key, split):
    wl = WORKLOADS[key]
    run = _oracle_run(wl, wl.chunk)
    _check_attention(ops, wl, run, run["blocks"], split=split)


@pytest.mark.parametrize("key", SMALL_SPARSE)
def test_attention_staged_dense_call(ops, key):
    # block_idx == NULL: every history block
    wl = WORKLOADS[key]
    run = _oracle_run(wl, wl.chunk)
    _check_attention(ops, wl, run, None)


def test_attention_staged_c2_full_size_sampled(ops):
    wl = WORKLOADS["c2"]
    heads = [3, 10]
    run = _oracle_run(wl, wl.chunk, heads)
    rows = sample_rows(wl, 2, np.random.default_rng(1))
    _check_attention(ops, _sub(wl, heads), run, None, rows, split=True)


def test_attention_staged_c4_full_size_sampled(ops):
    wl = WORKLOADS["c4"]
    heads = [7]
    run = _oracle_run(wl, wl.chunk, heads)
    rows = sample_rows(wl, 2, np.random.default_rng(2))
    _check_attention(ops, _sub(wl, heads), run, run["blocks"], rows)


# ---- whole path --------------------------------------------------------------------------

def _gpu_stream(ops, wl, upto, t_begin=0, heads=None, record=()):
    """Run the fused chunk call for chunks 1..upto; returns outputs of `record` chunks."""
    import torch
    wlh = _sub(wl, heads)
    shp = shape_of(wlh)
    tabs = _tables(ops, wl, t_begin)
    cache = ops.DeviceKVCache(shp, wl.window, t_begin)
    centres = key_centres(wl, 0) if wl.keys == "clustered" else None
    res = {}
    for c in range(1, upto + 1):
        x = inputs(wl, c, 0, heads, centres)
        t0 = wl.t0_of(c) + t_begin
        k_f, k_b = lib_budget(wl, c, t_begin)
        if wl.dense:
            k_f, k_b = -1, 0
        ws = torch.empty(ops.chunk_workspace_bytes(shp, k_f, k_b), dtype=torch.uint8, device="cuda")
        out = torch.empty((wlh.B, wlh.Lq, wlh.H, wlh.D), dtype=torch.bfloat16, device="cuda")
        ops.chunk_attention(to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"]), cache, tabs, t0, k_f, k_b, ws, out)
        if c in record or c == upto:
            torch.cuda.synchronize()
            res[c] = (from_dev(out), ws, k_f, k_b)
    assert ops.device_status() == 0
    return res, cache


def _e2e_compare(wl, run, gpu_out, blocks=None, rows=None):
    """Output of the fused call vs the oracle over every compared row. ``blocks``
    are the key sets to attend (default: the oracle's selection); where the
    GPU's selection differed validly at a near-tie, :func:`_e2e_selection`
    substitutes the GPU's own lists so that those rows are compared too."""
    use = run["blocks"] if blocks is None else blocks
    o_want, _ = o_path.attend_chunk(run["q_rot"], run["cache"], run["t0"], wl.Fc, use, rows)
    got = bits_to_f64(gpu_out)
    sel = np.arange(wl.Lq) if rows is None else rows
    return attn_errors(got[:, sel], o_want[:, sel])


def _e2e_selection(wl, run, ws, k_f, k_b, heads=None, max_near=0.02):
    """Checks the fused call's selection against the oracle (:func:`check_selection`)
    and returns the key sets its attention used."""
    kfe = run["frames"].shape[-1]
    fr, bl, ct = ws_lists(wl, ws, k_f, k_b, kfe)
    if heads is not None:
        fr, bl, ct = fr[:, heads], bl[:, heads], ct[:, heads]
    n, bad, near, blocks = check_selection(run, fr, bl, ct)
    assert bad == 0 and near <= max_near * n, (bad, near, n)
    return blocks


@pytest.mark.parametrize("key", SMALL)
def test_chunk_attention_end_to_end(ops, key):
    wl = WORKLOADS[key]
    res, _ = _gpu_stream(ops, wl, wl.chunk)
    out, ws, k_f, k_b = res[wl.chunk]
    run = _oracle_run(wl, wl.chunk)
    blocks = None
    if not wl.dense and k_b > 0:
        blocks = _e2e_selection(wl, run, ws, k_f, k_b)
    mx, mean, rel = _e2e_compare(wl, run, out, blocks)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean, rel)


def test_chunk_attention_global_time_shift(ops):
    # the same stream started at global frame 100: identical outputs up to
    # rounding of the rotated values, and parity with the oracle
    wl = WORKLOADS["c1s"]
    a, _ = _gpu_stream(ops, wl, wl.chunk, 0)
    b, _ = _gpu_stream(ops, wl, wl.chunk, 100)
    run = _oracle_run(wl, wl.chunk, None, 100)
    mx, mean, _ = _e2e_compare(wl, run, b[wl.chunk][0])
    assert mx <= MAX_ABS and mean <= MEAN_ABS
    d = np.abs(bits_to_f64(a[wl.chunk][0]) - bits_to_f64(b[wl.chunk][0]))
    assert d.max() <= 2 * MAX_ABS


def test_chunk_attention_rolling_window_wrap(ops):
    # window of 8 frames over 7 chunks of 3: slots wrap twice
    wl = WORKLOADS["r64s"].with_chunk(7)
    res, cache = _gpu_stream(ops, wl, 7)
    out, ws, k_f, k_b = res[7]
    run = _oracle_run(wl, 7)
    assert cache.history_frames(run["t0"]) == (13, 5)
    blocks = _e2e_selection(wl, run, ws, k_f, k_b)
    mx, mean, _ = _e2e_compare(wl, run, out, blocks)
    assert mx <= MAX_ABS and mean <= MEAN_ABS


def test_chunk_attention_first_chunk_has_no_history(ops):
    wl = WORKLOADS["r128"].with_chunk(1)
    res, _ = _gpu_stream(ops, wl, 1)
    run = _oracle_run(wl, 1)
    mx, mean, _ = _e2e_compare(wl, run, res[1][0])
    assert mx <= MAX_ABS and mean <= MEAN_ABS


def test_c2_dense_end_to_end_sampled(ops):
    wl = WORKLOADS["c2"]
    res, _ = _gpu_stream(ops, wl, wl.chunk)
    heads = [0, 11]
    run = _oracle_run(wl, wl.chunk, heads)
    rows = sample_rows(wl, 1, np.random.default_rng(3))
    out = res[wl.chunk][0][:, :, heads]
    mx, mean, rel = _e2e_compare(_sub(wl, heads), run, out, None, rows)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean, rel)


@pytest.mark.parametrize("chunk", [2, 7])
def test_c3_hsa_end_to_end_sampled(ops, chunk):
    wl = WORKLOADS["c3"].with_chunk(chunk)
    res, _ = _gpu_stream(ops, wl, chunk)
    out, ws, k_f, k_b = res[chunk]
    heads = [1, 6]
    run = _oracle_run(wl, chunk, heads)
    blocks = _e2e_selection(wl, run, ws, k_f, k_b, heads)
    rows = sample_rows(wl, 1, np.random.default_rng(4))
    mx, mean, rel = _e2e_compare(_sub(wl, heads), run, out[:, :, heads], blocks, rows)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean, rel)


def _ws_pairs(wl, ws, k_f, k_b):
    """The query-block pair table the fused call wrote into its workspace
    (after the counts in the layout of cva_chunk_workspace_bytes)."""
    d = wl
    bhq = d.B * d.H * d.NQB
    r256 = lambda x: (x + 255) // 256 * 256
    o_p = (r256(d.B * d.H * d.Fc * d.T_pad * d.D * 2) + r256(bhq * d.D * 4) + r256(bhq * max(k_f, 0) * 4)
           + r256(bhq * max(k_b, 0) * 4) + r256(bhq * 4))
    MT = -(-d.Fc * d.T_pad // 128)
    raw = ws.cpu().numpy()
    return raw[o_p:o_p + d.B * d.H * MT * 8].view(np.int32).reshape(d.B * d.H, MT, 2)


def test_query_block_pairs_are_mutual_best(ops):
    # c3 chunk 7: 18 history frames, 8 picked per query block, so the fused
    # call pairs the 64-row query blocks by shared frames before the attention
    wl = WORKLOADS["c3"].with_chunk(7)
    res, cache = _gpu_stream(ops, wl, 7)
    out, ws, k_f, k_b = res[7]
    _, F = cache.history_frames(wl.t0_of(7))
    kfe = min(k_f, F)
    assert wl.blk == 64 and F >= 2 * kfe
    fr, _, _ = ws_lists(wl, ws, k_f, k_b, kfe)
    fr = fr.reshape(wl.B * wl.H, wl.NQB, kfe)
    got = _ws_pairs(wl, ws, k_f, k_b)
    for bh in range(wl.B * wl.H):
        want = mutual_best_pairs(fr[bh])
        assert [tuple(int(v) for v in p) for p in got[bh, :len(want)]] == want, bh
        assert (got[bh, len(want):] == -1).all()
        ids = sorted(v for p in want for v in p if v >= 0)
        assert ids == list(range(wl.NQB))


def test_back_to_back_launches_match_staged_launches(ops):
    # Without stage events the fused call lets each kernel start while the
    # previous one drains (each waits for its inputs on the device); with
    # them, the kernels run one after another. The outputs are the same bits.
    import torch
    wl = WORKLOADS["c3"].with_chunk(7)
    res, cache = _gpu_stream(ops, wl, 7)
    out_chain, ws, k_f, k_b = res[7]
    x = inputs(wl, 7, 0, None, key_centres(wl, 0) if wl.keys == "clustered" else None)
    tabs = _tables(ops, wl, 0)
    out = torch.empty((wl.B, wl.Lq, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for e in evs:
        e.record()   # creates the underlying event
    ops.set_stage_events(evs)
    try:
        ops.chunk_attention(to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"]), cache, tabs, wl.t0_of(7),
                            k_f, k_b, ws, out)
        torch.cuda.synchronize()
    finally:
        ops.set_stage_events(None)
    assert ops.device_status() == 0
    assert np.array_equal(from_dev(out), out_chain)


@pytest.mark.parametrize("key", ["r64", "c1s"])
def test_rotate_append_pool_is_the_fused_calls_first_launch(ops, key):
    # steps 1-3 alone (plus the frame means) leave the same q_rot, pooled
    # queries and cache contents as the fused call's first launch
    import torch
    wl = WORKLOADS[key]
    shp = shape_of(wl)
    tabs = _tables(ops, wl)
    x = inputs(wl, 1, 0, None, key_centres(wl, 0) if wl.keys == "clustered" else None)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    fused = ops.DeviceKVCache(shp, wl.window, 0)
    ws = torch.zeros(ops.chunk_workspace_bytes(shp, -1, 0), dtype=torch.uint8, device="cuda")
    out = torch.empty((wl.B, wl.Lq, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    ops.chunk_attention(q, k, v, fused, tabs, wl.t0_of(1), -1, 0, ws, out)
    staged = ops.DeviceKVCache(shp, wl.window, 0)
    n_qrot = wl.B * wl.H * wl.Fc * wl.T_pad * wl.D
    q_rot = torch.empty(n_qrot, dtype=torch.bfloat16, device="cuda")
    qpool = torch.empty(wl.B * wl.H * wl.NQB * wl.D, dtype=torch.float32, device="cuda")
    ops.rotate_append_pool(q, k, v, staged, tabs, wl.t0_of(1), q_rot, qpool)
    ops.kv_frame_means(staged, wl.t0_of(1))
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    assert torch.equal(q_rot, ws[:n_qrot * 2].view(torch.bfloat16))
    for a, b in ((staged.k, fused.k), (staged.v, fused.v), (staged.kpool_blk, fused.kpool_blk)):
        assert torch.equal(a, b)
    torch.testing.assert_close(staged.kpool_frm, fused.kpool_frm, rtol=1e-6, atol=1e-6)
    # the dense first chunk does not pool its queries; the staged step-3 entry
    # pools the same rotated queries
    ref = torch.empty_like(qpool)
    ops.hsa_compress(q_rot, shp, ref)
    torch.cuda.synchronize()
    torch.testing.assert_close(qpool, ref, rtol=1e-6, atol=1e-6)


def test_chunk_call_replays_from_a_cuda_graph(ops):
    # The fused call (rotation, selection, pairing, attention, merge, the later
    # launches programmatic dependents) captured once into a CUDA graph and
    # replayed gives the eager call's bits.
    import torch
    wl = WORKLOADS["c3"].with_chunk(7)
    res, cache = _gpu_stream(ops, wl, 7)
    out_eager, ws, k_f, k_b = res[7]
    x = inputs(wl, 7, 0, None, key_centres(wl, 0) if wl.keys == "clustered" else None)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    tabs = _tables(ops, wl, 0)
    out = torch.empty((wl.B, wl.Lq, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        ops.chunk_attention(q, k, v, cache, tabs, wl.t0_of(7), k_f, k_b, ws, out)   # warm-up
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ops.chunk_attention(q, k, v, cache, tabs, wl.t0_of(7), k_f, k_b, ws, out)
    for _ in range(3):
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(from_dev(out), out_eager)
    assert ops.device_status() == 0


def test_c4_end_to_end_sampled(ops):
    wl = WORKLOADS["c4"]
    heads = [0, 21, 39]
    res, _ = _gpu_stream(ops, wl, wl.chunk)
    out, ws, k_f, k_b = res[wl.chunk]
    run = _oracle_run(wl, wl.chunk, heads)
    blocks = _e2e_selection(wl, run, ws, k_f, k_b, heads)
    rows = sample_rows(wl, 1, np.random.default_rng(5), blocks=range(0, wl.NQB, 3))
    mx, mean, rel = _e2e_compare(_sub(wl, heads), run, out[:, :, heads], blocks, rows)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean, rel)


def test_c5_streaming_window_sampled(ops):
    # 1.3B shape, rolling window of 60 frames: check chunk 21 (window full)
    # on two heads; the GPU runs every head of every chunk.
    wl = WORKLOADS["c5"].with_chunk(21)
    heads = [2, 9]
    res, cache = _gpu_stream(ops, wl, 21)
    out, ws, k_f, k_b = res[21]
    assert (k_f, k_b) == (20, 285)
    assert cache.history_frames(wl.t0_of(21)) == (3, 57)
    run = _oracle_run(wl, 21, heads)
    blocks = _e2e_selection(wl, run, ws, k_f, k_b, heads)
    rows = sample_rows(wl, 1, np.random.default_rng(6), blocks=range(0, wl.NQB, 4))
    mx, mean, rel = _e2e_compare(_sub(wl, heads), run, out[:, :, heads], blocks, rows)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean, rel)


# ---- top-p block budget ("Sparse VideoGen2", section B) --------------------------------------

def _topp_cap(wl, chunk, which, t_begin=0):
    """Cap of the top-p lists: every candidate block, or the chunk's top-k budget."""
    k_f, k_b = lib_budget(wl, chunk, t_begin)
    kfe = min(k_f, hist_count(wl, chunk, t_begin))
    return k_f, (kfe * wl.nb if which == "all" else k_b)


def _topp_compare(wl, run, gpu_blocks, gpu_cnt, p, cap, tol=1e-4):
    """Per (b, h, query block): identical to the oracle, or, where it differs,
    still a valid top-p choice under the oracle's own ranking (a prefix of it
    whose cut lies within `tol` of p in share, or at a score near-tie).
    Returns (units, mismatches that are not valid, valid mismatches, blocks):
    ``blocks`` is the oracle's lists with every validly differing unit's list
    replaced by the GPU's (padded with -1), the key sets the GPU attended."""
    B, H, NQB, _ = run["blocks"].shape
    blocks = run["blocks"].copy()
    bad = near = 0
    for b in range(B):
        for h in range(H):
            for qb in range(NQB):
                want = run["blocks"][b, h, qb]
                want = want[want >= 0]
                r = int(gpu_cnt[b, h, qb])
                got = gpu_blocks[b, h, qb, :max(r, 0)]
                if r == len(want) and np.array_equal(got, want):
                    continue
                if run["gap_f"][b, h, qb] < 1e-5:         # the frames themselves were a near tie
                    near += 1
                    blocks[b, h, qb] = -1
                    blocks[b, h, qb, :r] = got
                    continue
                ft = run["frames"][b, h, qb]
                kb = np.stack([run["cache"].frames[t]["kb"][b, h] for t in ft])
                ids, sc, above = o_hsa.topp_ranking(run["qbar_blk"][b, h, qb], kb, ft, wl.nb, wl.T_f, wl.blk)
                lim = min(cap, len(ids))
                ok = 1 <= r <= lim
                if ok and not np.array_equal(np.sort(ids[:r]), got):
                    ok = r < len(ids) and o_hsa.rel_gap(sc[r - 1], sc[r]) < 1e-5
                if ok and r > 1 and above[r - 1] >= p + tol:
                    ok = False                               # took a block it should not have
                if ok and r < lim and above[r] < p - tol:
                    ok = False                               # stopped before reaching p
                if ok:
                    near += 1
                    blocks[b, h, qb] = -1
                    blocks[b, h, qb, :r] = got
                else:
                    bad += 1
    return B * H * NQB, bad, near, blocks


def _staged_select_topp(ops, wl, run, p, cap):
    import torch
    cache = _gpu_cache_from_oracle(ops, wl, run)
    qd = to_dev(f64_to_bits(_head_major(wl, run["q_rot"])))
    pb = torch.empty((wl.B, wl.H, wl.NQB, wl.D), dtype=torch.float32, device="cuda")
    ops.hsa_compress(qd, shape_of(wl), pb)
    kfe = run["frames"].shape[-1]
    fi = torch.full((wl.B, wl.H, wl.NQB, max(kfe, 1)), -7, dtype=torch.int32, device="cuda")
    bi = torch.full((wl.B, wl.H, wl.NQB, cap), -7, dtype=torch.int32, device="cuda")
    bc = torch.full((wl.B, wl.H, wl.NQB), -7, dtype=torch.int32, device="cuda")
    ops.hsa_select_topp(pb, cache, run["t0"], run["k_f"], cap, p, fi, bi, bc)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    return fi.cpu().numpy(), bi.cpu().numpy(), bc.cpu().numpy()


@pytest.mark.parametrize("p", [0.5, 0.9])
@pytest.mark.parametrize("key", SMALL_SPARSE)
def test_hsa_select_topp_staged(ops, key, p):
    wl = WORKLOADS[key]
    _, cap = _topp_cap(wl, wl.chunk, "all")
    run = _oracle_run(wl, wl.chunk, topp=p, cap=cap)
    fi, bi, bc = _staged_select_topp(ops, wl, run, p, cap)
    assert np.all((bc >= 1) & (bc <= cap))
    n, bad, near, _ = _topp_compare(wl, run, bi, bc, p, cap)
    assert bad == 0 and near <= 0.05 * n, (bad, near, n)
    kfe = run["frames"].shape[-1]
    ok = run["gap_f"] >= 1e-5
    np.testing.assert_array_equal(fi[..., :kfe][ok], run["frames"][ok])


def test_hsa_select_topp_cap_binds(ops):
    # p close to 1 with the cap at the top-k budget: every list is the top-k
    wl = WORKLOADS["r128"]
    _, cap = _topp_cap(wl, wl.chunk, "budget")
    run = _oracle_run(wl, wl.chunk, topp=0.999, cap=cap)
    _, bi, bc = _staged_select_topp(ops, wl, run, 0.999, cap)
    n, bad, near, _ = _topp_compare(wl, run, bi, bc, 0.999, cap)
    assert bad == 0 and near <= 0.05 * n, (bad, near, n)
    runk = _oracle_run(wl, wl.chunk)
    full = np.all(run["blocks"] >= 0, axis=-1)
    assert full.mean() > 0.9
    np.testing.assert_array_equal(run["blocks"][full], runk["blocks"][full])


@pytest.mark.parametrize("chunk,p", [(4, 0.9), (7, 0.7)])
def test_hsa_select_topp_c3_full_size(ops, chunk, p):
    wl = WORKLOADS["c3"].with_chunk(chunk)
    heads = [0, 5, 11]
    _, cap = _topp_cap(wl, chunk, "all")
    run = _oracle_run(wl, chunk, heads, topp=p, cap=cap)
    fi, bi, bc = _staged_select_topp(ops, _sub(wl, heads), run, p, cap)
    n, bad, near, _ = _topp_compare(_sub(wl, heads), run, bi, bc, p, cap)
    assert bad == 0 and near <= 0.05 * n, (bad, near, n)


def _gpu_stream_topp(ops, wl, upto, p, which):
    """Fused top-p chunk calls for chunks 2..upto (chunk 1 dense); returns the
    last chunk's output, its block lists and counts."""
    import torch
    shp = shape_of(wl)
    tabs = _tables(ops, wl)
    cache = ops.DeviceKVCache(shp, wl.window, 0)
    centres = key_centres(wl, 0) if wl.keys == "clustered" else None
    for c in range(1, upto + 1):
        x = inputs(wl, c, 0, None, centres)
        out = torch.empty((wl.B, wl.Lq, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
        args = [to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"]), cache, tabs, wl.t0_of(c)]
        if c == 1:
            ws = torch.empty(ops.chunk_workspace_bytes(shp, -1, 0), dtype=torch.uint8, device="cuda")
            ops.chunk_attention(*args, -1, 0, ws, out)
            continue
        k_f, cap = _topp_cap(wl, c, which)
        ws = torch.empty(ops.chunk_workspace_bytes(shp, k_f, cap), dtype=torch.uint8, device="cuda")
        ops.chunk_attention_topp(*args, k_f, cap, p, ws, out)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    kfe = min(k_f, hist_count(wl, upto))
    _, gb, gc = ws_lists(wl, ws, k_f, cap, kfe)
    return from_dev(out), gb, gc, cap


@pytest.mark.parametrize("key,p", [("c1s", 0.6), ("r64", 0.8), ("r128", 0.5), ("r64s", 0.9)])
def test_chunk_attention_topp_end_to_end(ops, key, p):
    wl = WORKLOADS[key]
    out, gb, gc, cap = _gpu_stream_topp(ops, wl, wl.chunk, p, "all")
    run = _oracle_run(wl, wl.chunk, topp=p, cap=cap)
    n, bad, near, blocks = _topp_compare(wl, run, gb, gc, p, cap)
    assert bad == 0 and near <= 0.05 * n, (bad, near, n)
    mx, mean, rel = _e2e_compare(wl, run, out, blocks)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean, rel)


def test_c3_topp_end_to_end_sampled(ops):
    wl = WORKLOADS["c3"].with_chunk(7)
    p = 0.9
    out, gb, gc, cap = _gpu_stream_topp(ops, wl, 7, p, "all")
    heads = [1, 6]
    run = _oracle_run(wl, 7, heads, topp=p, cap=cap)
    gb, gc = gb[:, heads], gc[:, heads]
    n, bad, near, blocks = _topp_compare(_sub(wl, heads), run, gb, gc, p, cap)
    assert bad == 0 and near <= 0.05 * n, (bad, near, n)
    rows = sample_rows(wl, 1, np.random.default_rng(7))
    mx, mean, rel = _e2e_compare(_sub(wl, heads), run, out[:, :, heads], blocks, rows)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean, rel)


@pytest.mark.parametrize("key", ["c1s", "r64", "r128"])
def test_chunk_call_writes_frame_means(ops, key):
    # the fused call computes the new frames' frame means in the attention
    # launch: equal to the token means of the stored keys
    wl = WORKLOADS[key]
    _, cache = _gpu_stream(ops, wl, wl.chunk)
    kc = bits_to_f64(from_dev(cache.k))
    got = cache.kpool_frm.cpu().numpy().astype(np.float64)
    for f in range(wl.Fc):
        slot = (wl.t0 + f) % wl.window
        want = o_hsa.frame_mean(kc[:, :, slot, :wl.T_f])
        np.testing.assert_allclose(got[:, :, slot], want, rtol=0, atol=2e-6 * max(1.0, np.abs(want).max()))


# ---- denoising steps of a chunk -----------------------------------------------------------

def test_denoising_passes_leave_no_trace(ops):
    # chunk 3 runs two noisy passes (other inputs) before its clean pass;
    # every output from the clean pass on is bit-identical to a stream without them
    import torch
    wl = WORKLOADS["r64s"].with_chunk(5)
    shp = shape_of(wl)
    tabs = _tables(ops, wl)

    def run(noisy):
        cache = ops.DeviceKVCache(shp, wl.window, 0)
        outs = {}
        for c in range(1, 6):
            k_f, k_b = lib_budget(wl, c)
            ws = torch.empty(ops.chunk_workspace_bytes(shp, k_f, k_b), dtype=torch.uint8, device="cuda")
            layers = [11 + i for i in range(noisy if c == 3 else 0)] + [0]
            for layer in layers:
                x = inputs(wl, c, layer)
                out = torch.empty((wl.B, wl.Lq, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
                ops.chunk_attention(to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"]), cache, tabs, wl.t0_of(c),
                                    k_f, k_b, ws, out)
            outs[c] = from_dev(out)
        torch.cuda.synchronize()
        assert ops.device_status() == 0
        return outs

    a, b = run(0), run(2)
    for c in (3, 4, 5):
        np.testing.assert_array_equal(a[c], b[c])


# ---- edge cases and errors ------------------------------------------------------------------

def test_zero_blocks_attends_current_chunk_only(ops):
    wl = WORKLOADS["r64"]
    run = _oracle_run(wl, wl.chunk)
    empty = np.zeros(run["blocks"].shape[:-1] + (0,), dtype=np.int64)
    _check_attention(ops, wl, run, empty)


def test_single_block_budget(ops):
    wl = WORKLOADS["r128"]
    run = _oracle_run(wl, wl.chunk)
    sel = o_path.select_chunk(run["qbar_blk"], run["cache"], run["cache"].history(run["t0"], wl.Fc), 1, 1)
    _check_attention(ops, wl, run, sel[1])


def test_bad_block_index_is_latched_not_read(ops):
    import torch
    wl = WORKLOADS["r64"]
    run = _oracle_run(wl, wl.chunk)
    cache = _gpu_cache_from_oracle(ops, wl, run)
    qd = to_dev(f64_to_bits(_head_major(wl, run["q_rot"])))
    blocks = run["blocks"].astype(np.int32).copy()
    blocks[0, 0, 0, 0] = 10 ** 6          # far outside the cache window
    bi = torch.from_numpy(blocks).cuda()
    bc = torch.full(blocks.shape[:-1], blocks.shape[-1], dtype=torch.int32, device="cuda")
    out = torch.empty((wl.B, wl.Lq, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    ops.blocksparse_attn_fwd(qd, cache, run["t0"], bi, bc, blocks.shape[-1], out)
    torch.cuda.synchronize()
    assert ops.device_status(clear=True) == ops.DEV_BAD_INDEX
    assert ops.device_status() == 0


def test_bounded_wait_gives_up_and_latches_a_timeout(ops):
    # one CTA waits on an mbarrier nothing arrives at, with a 2 ms limit: the
    # wait returns, the timeout is latched and read back, the word clears, and
    # the context is still usable (a normal launch afterwards runs)
    import torch
    res = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    assert ops.device_status(clear=True) == 0
    ops.diag_wait_timeout(2000, res)
    torch.cuda.synchronize()
    assert res.cpu().tolist() == [1, 1]
    assert ops.device_status(clear=True) == ops.DEV_TIMEOUT
    assert ops.device_status() == 0
    with pytest.raises(ops.CvaError) as e:
        ops.diag_wait_timeout(0, res)
    assert e.value.code == ops.CVA_EINVAL
    y = torch.arange(8, dtype=torch.float32, device="cuda") + 1
    assert float(y.sum()) == 36.0


def test_mma_cycle_diagnostic_runs_and_checks_its_arguments(ops):
    import torch
    cycles = torch.zeros(4, dtype=torch.int64, device="cuda")
    ops.diag_mma_cycles(128, 128, 64, cycles)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    per = cycles.cpu().numpy() / (4 * 64)
    assert (per > 8).all() and (per < 10000).all(), per
    for m, n in ((96, 128), (128, 24), (64, 4), (128, 512)):
        with pytest.raises(ops.CvaError):
            ops.diag_mma_cycles(m, n, 64, cycles)


def test_host_errors(ops):
    import torch
    wl = WORKLOADS["r64"]
    shp = shape_of(wl)
    tabs = ops.DeviceRopeTables(wl.D, 8, wl.Fh, wl.Fw)
    cache = ops.DeviceKVCache(shp, wl.window)
    q = torch.zeros((wl.B, wl.Lq, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(ops.CvaError) as e:
        ops.chunk_attention(q, q, q, cache, tabs, 9, -1, 0, ws, out)   # t0 + Fc > max_t
    assert e.value.code == ops.CVA_ERANGE
    tabs2 = ops.DeviceRopeTables(wl.D, 64, wl.Fh, wl.Fw)
    with pytest.raises(ops.CvaError) as e:
        ops.chunk_attention(q, q, q, cache, tabs2, 6, -1, 0, ws, out)  # workspace too small
    assert e.value.code == ops.CVA_ENOMEM
    ws = torch.empty(ops.chunk_workspace_bytes(shp, 4, 9), dtype=torch.uint8, device="cuda")
    with pytest.raises(ops.CvaError) as e:
        ops.chunk_attention(q, q, q, cache, tabs2, 6, 4, 9, ws, out)   # k_b > k_f * nb = 8
    assert e.value.code == ops.CVA_ERANGE
    torch.cuda.synchronize()
    assert ops.device_status() == 0
