"""The head-sharded path: exchange plans and the whole chunk on gloo CPU ranks.

"Accelerating Video Generation Inference with Sequential-Parallel 3D
Positional Encoding Using a Global Time Index", sections 2A and 2C: tokens
sharded across ranks, one fused all-to-all of Q, K and V to a head-sharded
layout, one all-to-all back. The plans are checked by simulating the
exchange in one process for several rank counts; the class runs on two
gloo ranks with host stand-ins for the library copy and for the attention
(the oracle on the rank's heads), against the oracle on all heads.
"""
import multiprocessing as mp
import os
import socket
import sys
from datetime import timedelta

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.join(ROOT, "tests"))


def host_copy_rows(src, dst, n0, n1, inner, ss, ds):
    """Host version of cva_copy_rows_2d on flat uint8 arrays or tensors."""
    for i0 in range(n0):
        for i1 in range(n1):
            so = i0 * ss[0] + i1 * ss[1]
            do = i0 * ds[0] + i1 * ds[1]
            dst[do:do + inner] = src[so:so + inner]


def _simulate(B, Lq, H, D, P, rng):
    """Full-size tensors, each rank's slice packed, exchanged, unpacked."""
    from autoregressive_video_dit_b200.sharded import ShardPlan
    pl = ShardPlan(B, Lq, H, D, P)
    full = [rng.integers(0, 65535, (B, Lq, H, D), dtype=np.uint16) for _ in range(3)]
    L, Hl = pl.L, pl.Hl
    send = []
    for r in range(P):
        buf = np.zeros(3 * pl.slab * P, np.uint8)
        for t in range(3):
            x = np.ascontiguousarray(full[t][:, r * L:(r + 1) * L]).view(np.uint8).reshape(-1)
            n0, n1, inner, ss, ds, so, do = pl.pack(t)
            host_copy_rows(x[so:], buf[do:], n0, n1, inner, ss, ds)
        send.append(buf.reshape(P, -1))
    recv = [np.concatenate([send[s][r] for s in range(P)]) for r in range(P)]   # all-to-all
    for r in range(P):
        for t in range(3):
            loc = np.zeros((B, Lq, Hl, D), np.uint16)
            n0, n1, inner, ss, ds, so, do = pl.unpack(t)
            host_copy_rows(recv[r][so:], loc.view(np.uint8).reshape(-1)[do:], n0, n1, inner, ss, ds)
            np.testing.assert_array_equal(loc, full[t][:, :, r * Hl:(r + 1) * Hl])
    # output path: rank r holds heads r*Hl.. for all tokens; it returns token slices
    outs = rng.integers(0, 65535, (B, Lq, H, D), dtype=np.uint16)
    send2 = []
    for r in range(P):
        o = np.ascontiguousarray(outs[:, :, r * Hl:(r + 1) * Hl]).view(np.uint8).reshape(-1)
        buf = np.zeros(pl.slab * P, np.uint8)
        n0, n1, inner, ss, ds, so, do = pl.pack_out()
        host_copy_rows(o[so:], buf[do:], n0, n1, inner, ss, ds)
        send2.append(buf.reshape(P, -1))
    for r in range(P):
        recv2 = np.concatenate([send2[s][r] for s in range(P)])
        got = np.zeros((B, L, H, D), np.uint16)
        n0, n1, inner, ss, ds, so, do = pl.unpack_out()
        host_copy_rows(recv2[so:], got.view(np.uint8).reshape(-1)[do:], n0, n1, inner, ss, ds)
        np.testing.assert_array_equal(got, outs[:, r * L:(r + 1) * L])


@pytest.mark.parametrize("B,Lq,H,D,P", [(1, 12, 4, 8, 1), (1, 12, 4, 8, 2), (2, 12, 6, 8, 3),
                                        (1, 24, 8, 16, 4), (2, 8, 4, 8, 4)])
def test_exchange_plans_move_every_row_to_its_rank(B, Lq, H, D, P):
    _simulate(B, Lq, H, D, P, np.random.default_rng(B * 100 + P))


def test_plan_rejects_uneven_splits():
    from autoregressive_video_dit_b200.sharded import ShardPlan
    with pytest.raises(ValueError):
        ShardPlan(1, 10, 4, 8, 3)      # tokens
    with pytest.raises(ValueError):
        ShardPlan(1, 12, 6, 8, 4)      # heads
    with pytest.raises(ValueError):
        ShardPlan(1, 12, 2, 4, 2)      # 8-byte head groups


# ---- the class on two gloo ranks ------------------------------------------------------------

def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _OracleHeads:
    """The oracle path on one rank's heads, fed and read as bf16 tensors."""

    def __init__(self, wl, heads):
        from oracle import path as o_path
        self.o_path = o_path
        self.wl = wl
        self.cache = o_path.FrameCache(wl.B, heads, wl.D, wl.T_f, wl.blk, wl.window)

    def __call__(self, q, k, v, t0, k_f, k_b, out):
        import torch
        from _util import bits_to_f64, f64_to_bits
        wl = self.wl
        x = [bits_to_f64(a.view(torch.int16).numpy().view(np.uint16)) for a in (q, k, v)]
        run = self.o_path.run_chunk(self.cache, *x, Fh=wl.Fh, Fw=wl.Fw, Fc=wl.Fc, t0=t0, k_f=k_f, k_b=k_b,
                                    dense=k_f < 0, store="bf16")
        o = self.o_path.round_bf16(run["o"])
        out.copy_(torch.from_numpy(f64_to_bits(o).view(np.int16)).view(torch.bfloat16))


def _sharded_rank(rank, world, port, key, res):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    try:
        from autoregressive_video_dit_b200 import ops
        from autoregressive_video_dit_b200.sharded import HeadShardedChunkAttention
        from cva_workload import WORKLOADS, chunk_inputs
        from _util import oracle_budget
        wl = WORKLOADS[key]
        shape = ops.make_shape(wl.B, wl.H, wl.D, wl.Fh, wl.Fw, wl.Fc, wl.blk)
        Hl = wl.H // world
        path = HeadShardedChunkAttention(shape, wl.window, None, device="cpu", copy_rows=host_copy_rows,
                                         attend=_OracleHeads(wl, Hl))
        L = wl.Lq // world
        for c in range(1, wl.chunk + 1):
            x = chunk_inputs(wl, c)
            sl = [torch.from_numpy(np.ascontiguousarray(x[n][:, rank * L:(rank + 1) * L]).view(np.int16))
                  .view(torch.bfloat16) for n in ("q", "k", "v")]
            k_f, k_b = oracle_budget(wl, c)
            if wl.dense:
                k_f, k_b = -1, 0
            out = torch.empty((wl.B, L, wl.H, wl.D), dtype=torch.bfloat16)
            path(*sl, wl.t0_of(c), k_f, k_b, out)
        res.put((rank, out.view(torch.int16).numpy().view(np.uint16).copy()))
    except Exception as e:  # report at once: the other rank then fails its next exchange
        res.put((rank, repr(e)))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("key", ["c1", "c1s"])
def test_head_sharded_chunks_on_two_ranks_equal_the_unsharded_oracle(key):
    from cva_workload import WORKLOADS, chunk_inputs
    from oracle import path as o_path
    from _util import bits_to_f64, f64_to_bits, oracle_budget
    wl = WORKLOADS[key]
    world = 2
    ctx = mp.get_context("spawn")
    res = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sharded_rank, args=(r, world, port, key, res)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        r, v = res.get(timeout=300)
        got[r] = v
        assert not isinstance(v, str), v
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the same chunks through the oracle on all heads at once
    cache = o_path.FrameCache(wl.B, wl.H, wl.D, wl.T_f, wl.blk, wl.window)
    for c in range(1, wl.chunk + 1):
        x = chunk_inputs(wl, c)
        k_f, k_b = oracle_budget(wl, c)
        run = o_path.run_chunk(cache, *(bits_to_f64(x[n]) for n in ("q", "k", "v")), Fh=wl.Fh, Fw=wl.Fw,
                               Fc=wl.Fc, t0=wl.t0_of(c), k_f=k_f, k_b=k_b, dense=wl.dense, store="bf16")
    want = f64_to_bits(o_path.round_bf16(run["o"]))
    L = wl.Lq // world
    for r in range(world):
        np.testing.assert_array_equal(got[r], want[:, r * L:(r + 1) * L])
