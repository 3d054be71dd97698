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
