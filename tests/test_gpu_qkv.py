"""The QKV projection fused with Causal-RoPE, the cache append and pooling.

"Accelerating Video Generation Inference with Sequential-Parallel 3D
Positional Encoding Using a Global Time Index", section 2C (operator
fusion). cva_qkv_rope_append is compared with the fp64 oracle (projection,
then the rotation of section 2B) on seeded hidden states and weights:
rotated q in the attention's padded layout, k and v in the cache slots,
pad rows zero, and the block / frame means of the stored values.
"""
import numpy as np
import pytest

from cva_workload import WORKLOADS, hidden_inputs
from oracle import hsa as o_hsa
from oracle import path as o_path
from oracle import qkv as o_qkv
from oracle import rope as o_rope
from _util import bits_to_f64, from_dev, rope_tol, shape_of, to_dev

pytestmark = pytest.mark.gpu


def _oracle_rows(wl, x64, w64, t0, rows):
    """q_rot, k_rot, v of the given token rows, [B, len(rows), H, D] (fp64)."""
    q, k, v = o_qkv.project(x64[:, rows], w64, wl.H, wl.D)
    t, h, w = o_rope.token_coords(wl.Fh, wl.Fw, wl.Fc, t0)
    ang = o_rope.pair_angles(wl.D, t[rows], h[rows], w[rows])
    rot = lambda a: np.transpose(o_rope.rotate(np.transpose(a, (0, 2, 1, 3)), ang), (0, 2, 1, 3))
    return rot(q), rot(k), v


def _check(key, hidden, rows=None):
    import torch
    from autoregressive_video_dit_b200 import ops

    wl = WORKLOADS[key]
    t0 = wl.t0
    inp = hidden_inputs(wl, hidden)
    x64, w64 = bits_to_f64(inp["x"]), bits_to_f64(inp["w"])
    tabs = ops.DeviceRopeTables(wl.D, t0 + wl.Fc, wl.Fh, wl.Fw)
    cache = ops.DeviceKVCache(shape_of(wl), wl.window, 0)
    q_rot = torch.full((wl.B, wl.H, wl.Fc * wl.T_pad, wl.D), float("nan"), dtype=torch.bfloat16, device="cuda")
    qpool = torch.full((wl.B, wl.H, wl.NQB, wl.D), float("nan"), dtype=torch.float32, device="cuda")
    ops.qkv_rope_append(to_dev(inp["x"]), to_dev(inp["w"]), cache, tabs, t0, q_rot, qpool)
    torch.cuda.synchronize()
    assert ops.device_status() == 0

    full = rows is None
    rows = np.arange(wl.Lq) if full else np.asarray(rows)
    q_o, k_o, v_o = _oracle_rows(wl, x64, w64, t0, rows)
    f = rows // wl.T_f
    rr = rows % wl.T_f
    slot = (t0 + f) % wl.window
    gq = bits_to_f64(from_dev(q_rot))                     # [B, H, Fc*T_pad, D]
    gk = bits_to_f64(from_dev(cache.k))                   # [B, H, W, T_pad, D]
    gv = bits_to_f64(from_dev(cache.v))
    got_q = np.transpose(gq[:, :, f * wl.T_pad + rr], (0, 2, 1, 3))
    got_k = np.transpose(gk[:, :, slot, rr], (0, 2, 1, 3))
    got_v = np.transpose(gv[:, :, slot, rr], (0, 2, 1, 3))
    for got, want in ((got_q, q_o), (got_k, k_o), (got_v, v_o)):
        err = np.abs(got - want)
        assert np.all(err <= rope_tol(want)), (err.max(), np.argmax(err))

    # pad rows of every frame are zero (q_rot and both cache tensors)
    pad = np.arange(wl.T_f, wl.T_pad)
    if pad.size:
        for fr in range(wl.Fc):
            assert np.all(gq[:, :, fr * wl.T_pad + pad] == 0)
            assert np.all(gk[:, :, (t0 + fr) % wl.window][:, :, pad] == 0)
            assert np.all(gv[:, :, (t0 + fr) % wl.window][:, :, pad] == 0)

    if full:
        # block means of the stored q and k, frame means of k (fp64 from the
        # oracle's values rounded to bf16; 2e-3 covers one-ulp rounding
        # differences of single elements)
        qr = o_path.round_bf16(q_o)                       # [B, Lq, H, D]
        kr = o_path.round_bf16(k_o)
        gp = qpool.cpu().numpy().astype(np.float64)
        gkb = cache.kpool_blk.cpu().numpy().astype(np.float64)
        gkf = cache.kpool_frm.cpu().numpy().astype(np.float64)
        for fr in range(wl.Fc):
            seg = slice(fr * wl.T_f, (fr + 1) * wl.T_f)
            s = (t0 + fr) % wl.window
            qb = o_hsa.block_means(np.transpose(qr[:, seg], (0, 2, 1, 3)), wl.blk)   # [B, H, nb, D]
            kb = o_hsa.block_means(np.transpose(kr[:, seg], (0, 2, 1, 3)), wl.blk)
            np.testing.assert_allclose(gp[:, :, fr * wl.nb:(fr + 1) * wl.nb], qb, rtol=0, atol=2e-3)
            np.testing.assert_allclose(gkb[:, :, s], kb, rtol=0, atol=2e-3)
            kf = o_hsa.frame_mean(np.transpose(kr[:, seg], (0, 2, 1, 3)))
            np.testing.assert_allclose(gkf[:, :, s], kf, rtol=0, atol=2e-3)


@pytest.mark.parametrize("key,hidden", [("c1", 64), ("r64", 128), ("r128", 192), ("r64s", 64), ("c1s", 256),
                                        ("r64s", 320)])
def test_qkv_rope_append_small(key, hidden):
    _check(key, hidden)


def test_qkv_rope_append_c2_hidden1536_sampled():
    wl = WORKLOADS["c2"]
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([rng.integers(0, wl.Lq, 300), [0, wl.T_f - 1, wl.Lq - 1]]))
    _check("c2", 1536, rows)


def test_qkv_rope_append_c4_hidden5120_sampled():
    wl = WORKLOADS["c4"]
    rng = np.random.default_rng(4)
    rows = np.unique(np.concatenate([rng.integers(0, wl.Lq, 120), [0, wl.T_f - 1, wl.Lq - 1]]))
    _check("c4", 5120, rows)


def test_qkv_rope_append_rejects_bad_hidden():
    import torch
    from autoregressive_video_dit_b200 import ops
    wl = WORKLOADS["c1"]
    tabs = ops.DeviceRopeTables(wl.D, wl.t0 + wl.Fc, wl.Fh, wl.Fw)
    cache = ops.DeviceKVCache(shape_of(wl), wl.window, 0)
    x = torch.zeros((wl.B, wl.Lq, 96), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((3 * wl.H * wl.D, 96), dtype=torch.bfloat16, device="cuda")
    q_rot = torch.zeros((wl.B, wl.H, wl.Fc * wl.T_pad, wl.D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ops.CvaError):
        ops.qkv_rope_append(x, w, cache, tabs, wl.t0, q_rot)
    assert "multiple of 64" in ops.last_error()


# ---- whole path from the hidden states ----------------------------------------------------

def _oracle_stream_qkv(wl, hidden, w64, upto):
    """Oracle over chunks 1..upto fed by the projection (one weight for the
    layer): history appended as bf16 rotated k and bf16 v; returns the last
    chunk's path intermediates (selection, rotated q) without attention."""
    from _util import oracle_budget
    cache = o_path.FrameCache(wl.B, wl.H, wl.D, wl.T_f, wl.blk, wl.window)
    cache.t_begin = 0
    for c in range(1, upto + 1):
        x64 = bits_to_f64(hidden_inputs(wl, hidden, c)["x"])
        q, k, v = o_qkv.project(x64, w64, wl.H, wl.D)
        v = o_path.round_bf16(v)
        t0 = wl.t0_of(c)
        if c < upto:
            _, k_rot = o_path.rotate_chunk(q, k, wl.Fh, wl.Fw, wl.Fc, t0, "bf16")
            cache.append(k_rot, v, t0, wl.Fc)
            continue
        k_f, k_b = oracle_budget(wl, c)
        run = o_path.run_chunk(cache, q, k, v, Fh=wl.Fh, Fw=wl.Fw, Fc=wl.Fc, t0=t0, k_f=k_f, k_b=k_b,
                               dense=wl.dense, store="bf16", attend_too=False)
        run.update(cache=cache, t0=t0)
        return run


@pytest.mark.parametrize("key,hidden", [("c1", 128), ("c1s", 64), ("r64", 192), ("r128", 256), ("r64s", 128)])
def test_chunk_attention_from_hidden_states(key, hidden):
    import torch
    from autoregressive_video_dit_b200 import ops
    from _util import MAX_ABS, MEAN_ABS, attn_errors, lib_budget

    wl = WORKLOADS[key]
    upto = wl.chunk
    w_bits = hidden_inputs(wl, hidden, 1)["w"]      # one weight for the layer
    w64 = bits_to_f64(w_bits)
    shp = shape_of(wl)
    tabs = ops.DeviceRopeTables(wl.D, wl.t0_of(upto) + wl.Fc, wl.Fh, wl.Fw)
    cache = ops.DeviceKVCache(shp, wl.window, 0)
    wd = to_dev(w_bits)
    for c in range(1, upto + 1):
        k_f, k_b = (-1, 0) if wl.dense else lib_budget(wl, c)
        ws = torch.empty(ops.chunk_workspace_bytes(shp, k_f, k_b), dtype=torch.uint8, device="cuda")
        out = torch.empty((wl.B, wl.Lq, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
        ops.chunk_attention_qkv(to_dev(hidden_inputs(wl, hidden, c)["x"]), wd, cache, tabs, wl.t0_of(c),
                                k_f, k_b, ws, out)
    torch.cuda.synchronize()
    assert ops.device_status() == 0

    run = _oracle_stream_qkv(wl, hidden, w64, upto)
    o_want, _ = o_path.attend_chunk(run["q_rot"], run["cache"], run["t0"], wl.Fc, run["blocks"])
    got = bits_to_f64(from_dev(out))
    g, w = got, o_want
    if run["blocks"] is not None and k_b > 0:
        # query blocks whose selection differs from the oracle's (near ties) are left out
        bhq = wl.B * wl.H * wl.NQB
        r256 = lambda n: (n + 255) // 256 * 256
        off = r256(wl.B * wl.H * wl.Fc * wl.T_pad * wl.D * 2) + r256(bhq * wl.D * 4) + r256(bhq * max(k_f, 0) * 4)
        gb = ws[off:off + bhq * k_b * 4].cpu().numpy().view(np.int32).reshape(wl.B, wl.H, wl.NQB, k_b)
        ok = np.all(gb == run["blocks"], axis=-1)
        assert ok.mean() >= 0.98, ok.mean()
        sel = np.arange(wl.Lq)
        qb = (sel // wl.T_f) * wl.nb + (sel % wl.T_f) // wl.blk
        mask = np.transpose(ok[:, :, qb], (0, 2, 1))[..., None]
        g, w = np.where(mask, g, 0.0), np.where(mask, w, 0.0)
    mx, mean, rel = attn_errors(g, w)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean, rel)
