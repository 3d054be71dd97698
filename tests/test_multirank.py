"""Host logic of the multi-GPU run, exercised on CPU ranks (gloo, world size 2).

With N GPUs every rank runs its own independent instance of the path (its
own seeded layer): the job's step time is the slowest rank's, its work the
sum of the ranks'. These tests run that reduction over real process groups
of two CPU ranks, check that ranks draw distinct inputs, and that only rank
0 of the reference arm does work and prints.
"""
import json
import multiprocessing as mp
import os
import socket
import sys
from datetime import timedelta

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        ms, work = bench.reduce_over_ranks(1.5 + rank, 10.0 * (rank + 1), "cpu")
        # the end-to-end figure goes through the same reduction with no work
        e2e_ms, zero = bench.reduce_over_ranks(3.0 - rank, 0.0, "cpu")
        out.put((rank, ms, work, e2e_ms, zero))
    finally:
        dist.destroy_process_group()


def _run_ranks(world):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res)


def test_step_time_is_the_slowest_rank_and_work_adds_up():
    res = _run_ranks(2)
    for rank, ms, work, e2e_ms, zero in res:
        assert ms == 2.5            # max(1.5, 2.5)
        assert work == 30.0         # 10 + 20
        assert e2e_ms == 3.0        # max(3.0, 2.0)
        assert zero == 0.0


def test_without_a_process_group_values_pass_through():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_over_ranks(1.25, 7.0, "cpu") == (1.25, 7.0)


def test_ranks_draw_distinct_inputs():
    sys.path.insert(0, ROOT)
    import bench
    from cva_workload import WORKLOADS, chunk_inputs
    wl = WORKLOADS["c1"]
    layers = [bench.rank_layer(r) for r in range(4)]
    assert len(set(layers)) == 4
    xs = [chunk_inputs(wl, wl.chunk, layer)["q"] for layer in layers[:2]]
    assert xs[0].shape == xs[1].shape and not np.array_equal(xs[0], xs[1])


def test_reference_arm_runs_on_rank_zero_only(capsys, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--workload", "c1",
                                      "--steps", "1", "--warmup", "0"])
    assert bench.main() == 0
    assert capsys.readouterr().out == ""
    monkeypatch.setenv("RANK", "0")
    assert bench.main() == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_percentile_nearest_rank():
    sys.path.insert(0, ROOT)
    import bench
    xs = list(range(1, 101))
    assert bench.percentile(xs, 50) == 50 and bench.percentile(xs, 99) == 99
    assert bench.percentile([3.0], 99) == 3.0
