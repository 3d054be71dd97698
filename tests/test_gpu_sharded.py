"""The head-sharded path on the GPU.

cva_copy_rows_2d against numpy on random rows and strides; then the whole
head-sharded chunk call ("Accelerating Video Generation Inference with
Sequential-Parallel 3D Positional Encoding Using a Global Time Index",
sections 2A and 2C) with P ranks driven from one process on one GPU: each
rank's phases run through the library and the all-to-alls are done as
device copies between the ranks' buffers (no kernel waits on another
rank). The output is compared with the fp64 oracle run over all heads: each
rank's selection (read from its workspace) must equal the oracle's or be a
valid top-k at a near-tie, and the output must lie within the attention
tolerances of the oracle's attention over those selections. A single-rank
NCCL group must reproduce the unsharded call exactly.
"""
import os
import socket

import numpy as np
import pytest

from cva_workload import WORKLOADS
from oracle import path as o_path
from _util import (MAX_ABS, MEAN_ABS, attn_errors, bits_to_f64, check_selection, from_dev, hist_count, inputs,
                   lib_budget, oracle_run, sample_rows, shape_of, to_dev, ws_lists)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n0,n1,inner,pad", [(5, 3, 16, 0), (7, 4, 256, 32), (3, 9, 1024, 16), (1, 1, 48, 0)])
def test_copy_rows_2d_matches_numpy(n0, n1, inner, pad):
    import torch
    from autoregressive_video_dit_b200 import ops
    rng = np.random.default_rng(n0 * 31 + n1)
    ss = ((n1 * inner + pad), inner)            # source rows [n0][n1], padded per i0
    ds = (inner, (n0 * inner + pad))            # destination [n1][n0], padded per i1
    src = rng.integers(0, 256, n0 * ss[0] + 64, dtype=np.uint8)
    dst0 = rng.integers(0, 256, n1 * ds[1] + 64, dtype=np.uint8)
    want = dst0.copy()
    for i0 in range(n0):
        for i1 in range(n1):
            want[i0 * ds[0] + i1 * ds[1]:][:inner] = src[i0 * ss[0] + i1 * ss[1]:][:inner]
    s = torch.from_numpy(src).cuda()
    d = torch.from_numpy(dst0).cuda()
    ops.copy_rows_2d(s, d, n0, n1, inner, ss, ds)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(d.cpu().numpy(), want)


def test_copy_rows_2d_rejects_misaligned():
    import torch
    from autoregressive_video_dit_b200 import ops
    s = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ops.CvaError):
        ops.copy_rows_2d(s, s[128:], 2, 2, 24, (48, 24), (24, 48))


def _unsharded(ops, wl, upto, tabs):
    import torch
    shp = shape_of(wl)
    cache = ops.DeviceKVCache(shp, wl.window, 0)
    for c in range(1, upto + 1):
        x = inputs(wl, c)
        k_f, k_b = (-1, 0) if wl.dense else lib_budget(wl, c)
        ws = torch.empty(ops.chunk_workspace_bytes(shp, k_f, k_b), dtype=torch.uint8, device="cuda")
        out = torch.empty((wl.B, wl.Lq, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
        ops.chunk_attention(to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"]), cache, tabs, wl.t0_of(c), k_f, k_b,
                            ws, out)
    torch.cuda.synchronize()
    return from_dev(out)


@pytest.mark.parametrize("key,P,upto", [("c1s", 2, None), ("r64", 2, None), ("c3", 3, 4)])
def test_head_sharded_ranks_match_the_oracle(key, P, upto):
    import torch
    from autoregressive_video_dit_b200 import ops
    from autoregressive_video_dit_b200.sharded import HeadShardedChunkAttention
    wl = WORKLOADS[key].with_chunk(upto) if upto else WORKLOADS[key]
    upto = wl.chunk
    shp = shape_of(wl)
    tabs = ops.DeviceRopeTables(wl.D, wl.t0_of(upto) + wl.Fc, wl.Fh, wl.Fw)
    ranks = [HeadShardedChunkAttention(shp, wl.window, tabs, rank=r, world=P) for r in range(P)]
    L = wl.Lq // P
    for c in range(1, upto + 1):
        x = inputs(wl, c)
        k_f, k_b = (-1, 0) if wl.dense else lib_budget(wl, c)
        # each rank's budget is over its own heads' history: the same numbers
        sends = [rk.pack(*(to_dev(np.ascontiguousarray(x[n][:, r * L:(r + 1) * L])) for n in ("q", "k", "v")))
                 for r, rk in enumerate(ranks)]
        recvs = [torch.cat([s.view(P, -1)[r] for s in sends]) for r in range(P)]          # all-to-all
        sends2 = [rk.compute(recvs[r], wl.t0_of(c), k_f, k_b) for r, rk in enumerate(ranks)]
        recvs2 = [torch.cat([s.view(P, -1)[r] for s in sends2]) for r in range(P)]        # all-to-all
        outs = []
        for r, rk in enumerate(ranks):
            o = torch.empty((wl.B, L, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
            rk.finish(recvs2[r], o)
            outs.append(o)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    got = np.concatenate([from_dev(o) for o in outs], axis=1)

    run = oracle_run(wl, upto)
    blocks = None
    if not wl.dense and k_b > 0:
        # the ranks' selections, head groups side by side
        kfe = min(k_f, hist_count(wl, upto))
        loc = WORKLOADS[key].replace(H=wl.H // P)
        lists = [ws_lists(loc, rk.ws, k_f, k_b, kfe) for rk in ranks]
        fr, bl, ct = (np.concatenate([li[i] for li in lists], axis=1) for i in range(3))
        n, bad, near, blocks = check_selection(run, fr, bl, ct)
        assert bad == 0 and near <= 0.02 * n, (bad, near, n)
    rows = sample_rows(wl, 2, np.random.default_rng(11)) if wl.Lq > 1000 else None
    o_want, _ = o_path.attend_chunk(run["q_rot"], run["cache"], run["t0"], wl.Fc,
                                    run["blocks"] if blocks is None else blocks, rows)
    sel = np.arange(wl.Lq) if rows is None else rows
    mx, mean, rel = attn_errors(bits_to_f64(got)[:, sel], o_want[:, sel])
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean, rel)


def test_single_rank_nccl_group_equals_the_unsharded_call():
    import torch
    import torch.distributed as dist
    from autoregressive_video_dit_b200 import ops
    from autoregressive_video_dit_b200.sharded import HeadShardedChunkAttention
    wl = WORKLOADS["c1s"]
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        shp = shape_of(wl)
        tabs = ops.DeviceRopeTables(wl.D, wl.t0_of(wl.chunk) + wl.Fc, wl.Fh, wl.Fw)
        path = HeadShardedChunkAttention(shp, wl.window, tabs)
        for c in range(1, wl.chunk + 1):
            x = inputs(wl, c)
            k_f, k_b = lib_budget(wl, c)
            out = torch.empty((wl.B, wl.Lq, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
            path(to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"]), wl.t0_of(c), k_f, k_b, out)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(from_dev(out), _unsharded(ops, wl, wl.chunk, tabs))
    finally:
        dist.destroy_process_group()
