#!/usr/bin/env python
"""Benchmark of the per-chunk attention path on B200.

One step = one chunk through the whole path (rotary embedding with the
global time index, cache append, pooling, selection when the budget is
sparse, block-sparse attention) via ``cva_chunk_attention``, with the
chunk's Q/K/V already resident in HBM and the history already in the cache.
L2 is flushed before every step (a 256 MiB write, then a 256 MiB read of
another buffer so that no dirty line of the flush is left to be written
back inside the timed step) and only the step itself is timed (CUDA events
on the launching stream).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c4]
    python bench.py --impl reference      # the fp64 oracle on the host cores

Prints one JSON line (rank 0). The line's workload is c4 (the 14B-shaped
720P chunk with hierarchical selection, the largest single-GPU
configuration); on one GPU the line also carries ``per_config`` entries
measured in the same run: c2 (1.3B-shaped dense chunk), c3 chunk 7 (1.3B
shape, hierarchical selection) and c5 (80 chunks x 30 layers streamed
through a rolling window, per-chunk latency p50/p99). With N > 1
(torchrun) every rank runs its own independent instance of the line's
workload (its own seeded layer): weak scaling, no data-path collective; the
reported time is the max over ranks, and the per-config entries are left
out.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "chunk attention latency (ms) and effective TFLOP/s, % of B200 bf16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--workload", default="c4")
    ap.add_argument("--chunk", type=int, default=None, help="chunk index (default: the workload's)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per_config entries (c2 dense, c3 chunk 7, c5 streaming) of the line")
    ap.add_argument("--sweep", action="store_true",
                    help="chunks 1..N of the workload under its literal and mirrored density "
                         "schedules, one JSON line each (measurement mode, not the bench line)")
    ap.add_argument("--stream", action="store_true",
                    help="streaming run: every chunk of the workload through all its layers, "
                         "per-chunk latency percentiles (measurement mode, not the bench line)")
    ap.add_argument("--qkv", action="store_true",
                    help="the QKV projection fused with rotation/append/pooling (hidden = H*D) "
                         "against cuBLAS GEMMs followed by the separate kernels (measurement mode)")
    ap.add_argument("--mma-shapes", action="store_true",
                    help="tensor-core time of one tcgen05.mma per shape (64- and 128-row tiles), "
                         "one JSON line each (measurement mode)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def host_cores():
    try:
        n_aff = len(os.sched_getaffinity(0))
    except Exception:
        n_aff = os.cpu_count() or 1
    threads = n_aff
    try:
        from threadpoolctl import threadpool_info
        info = [i for i in threadpool_info() if i.get("user_api") == "blas"]
        if info:
            threads = max(int(i.get("num_threads", n_aff)) for i in info)
    except Exception:
        pass
    return n_aff, threads


# ---------------------------------------------------------------- workloads

def setup_workload(args, layer, wl=None):
    """Device state of one chunk: tables, cache with history, inputs, budget."""
    import numpy as np
    import torch
    from autoregressive_video_dit_b200 import ops
    from cva_workload import WORKLOADS, chunk_inputs, key_centres

    if wl is None:
        wl = WORKLOADS[args.workload]
        if args.chunk is not None:
            wl = wl.with_chunk(args.chunk)
    shape = ops.make_shape(wl.B, wl.H, wl.D, wl.Fh, wl.Fw, wl.Fc, wl.blk)
    tables = ops.DeviceRopeTables(wl.D, wl.t0 + wl.Fc, wl.Fh, wl.Fw)
    cache = ops.DeviceKVCache(shape, wl.window, 0)
    centres = key_centres(wl, layer) if wl.keys == "clustered" else None

    def dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)

    lo = max(0, wl.t0 + wl.Fc - wl.window)
    for c in range(lo // wl.Fc + 1, wl.chunk):
        x = chunk_inputs(wl, c, layer, centres=centres)
        ops.kv_append(dev(x["k"]), dev(x["v"]), cache, tables, wl.t0_of(c))
    x = chunk_inputs(wl, wl.chunk, layer, centres=centres)
    q, k, v = dev(x["q"]), dev(x["k"]), dev(x["v"])
    t_lo, F = cache.history_frames(wl.t0)
    if wl.dense:
        k_f, k_b = -1, 0
    else:
        k_f, k_b = ops.cag_budget(wl.chunk, F, wl.nb, dense=False, k_f_max=wl.k_f_max,
                                  d_base=(wl.d_base.numerator, wl.d_base.denominator),
                                  d_slope=(wl.d_slope.numerator, wl.d_slope.denominator),
                                  pivot=wl.d_pivot, k_b_fixed=wl.k_b_fixed)
    ws = torch.empty(ops.chunk_workspace_bytes(shape, k_f, k_b), dtype=torch.uint8, device="cuda")
    out = torch.empty((wl.B, wl.Lq, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    return dict(wl=wl, shape=shape, tables=tables, cache=cache, q=q, k=k, v=v, k_f=k_f, k_b=k_b,
                ws=ws, out=out, F=F, t_lo=t_lo, raw=x)


def attention_flops(st):
    """Algorithmic attention FLOPs of one chunk: 4*D*sum over (b, h, query
    block) of |valid queries| * |valid keys|, keys = picked history blocks'
    valid tokens plus the Lq tokens of the chunk."""
    import numpy as np
    wl = st["wl"]
    qcount = np.array([wl.blk] * (wl.nb - 1) + [wl.T_f - (wl.nb - 1) * wl.blk] * 1)
    qcount = np.tile(qcount, wl.Fc)                                   # [NQB]
    if st["k_f"] < 0 or st["F"] == 0:
        keys = st["F"] * wl.T_f + wl.Lq
        return 4.0 * wl.D * wl.B * wl.H * float(qcount.sum()) * keys
    blocks, cnt = block_lists(st)                                     # [B,H,NQB,k_b], [B,H,NQB]
    tail = wl.T_f - (wl.nb - 1) * wl.blk
    valid = np.where(blocks % wl.nb == wl.nb - 1, tail, wl.blk)
    valid = np.where(np.arange(st["k_b"]) < cnt[..., None], valid, 0)  # top-p lists are shorter
    keys = valid.sum(axis=-1) + wl.Lq                                 # [B,H,NQB]
    return 4.0 * wl.D * float((keys * qcount[None, None, :]).sum())


def block_lists(st):
    """Block lists and their lengths from the chunk workspace (its layout:
    rotated q, pooled q, frame lists, block lists, block counts)."""
    import numpy as np
    wl = st["wl"]
    bhq = wl.B * wl.H * wl.NQB
    r = lambda x: (x + 255) // 256 * 256
    off = (r(wl.B * wl.H * wl.Fc * wl.T_pad * wl.D * 2) + r(bhq * wl.D * 4)
           + r(bhq * max(st["k_f"], 0) * 4))
    raw = st["ws"][off:off + bhq * st["k_b"] * 4].cpu().numpy().view(np.int32)
    off += r(bhq * st["k_b"] * 4)
    cnt = st["ws"][off:off + bhq * 4].cpu().numpy().view(np.int32)
    return (raw.reshape(wl.B, wl.H, wl.NQB, st["k_b"]).astype(np.int64),
            cnt.reshape(wl.B, wl.H, wl.NQB).astype(np.int64))


def attention_launches(wl):
    """Launches of the attention step: the kernel, plus the merge of the
    tail-split pieces when the query tiles leave a partial last wave (the
    library's rule: tail = tiles mod SMs, pieces = min(SMs // tail, 160 //
    tail), split when pieces >= 2)."""
    import torch
    nsm = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    tiles = -(-wl.Fc * wl.T_pad // 128) * wl.B * wl.H
    tail = tiles % nsm
    pieces = min(nsm // tail, 160 // tail) if tail else 0
    return 2 if pieces >= 2 else 1


def rope_bytes(wl):
    """Algorithmic HBM bytes of the rotate/append/pool stage: read Q, K, V and
    write rotated Q, rotated K and V (bf16)."""
    return 6.0 * wl.Lq * wl.B * wl.H * wl.D * 2


# ---------------------------------------------------------------- clocks

REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


class ClockSampler:
    def __init__(self, enabled=True):
        self.proc = None
        self.path = None
        if not enabled:
            return
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        fd, self.path = tempfile.mkstemp(prefix="cva_clocks_", suffix=".csv")
        os.close(fd)
        q = "clocks.sm,clocks.max.sm,power.draw," + ",".join("clocks_event_reasons." + r for r in REASONS)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", *sel, "--query-gpu=" + q,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 3 + len(REASONS):
                    continue
                try:
                    rows.append((float(parts[0]), float(parts[1]), parts[3:3 + len(REASONS)]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        active = sorted({REASONS[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": active, "samples": len(rows)}


# ---------------------------------------------------------------- traffic record

def recorded_traffic(kernel_file, workload):
    """Per-launch DRAM bytes of the attention kernel from the committed ncu
    summary, if it was taken on the current source of that kernel."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    src = os.path.join(ROOT, "autoregressive_video_dit_b200", "csrc", kernel_file)
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    e = rec.get(workload, {}).get(kernel_file)
    if not e or e.get("source_sha") != sha:
        return None
    return e.get("bytes_per_launch")


# ---------------------------------------------------------------- CPU oracle timing

class OracleSample:
    """The fp64 oracle on one head of the chunk. The history is built once
    (untimed); each sample then times rotation, pooling and selection of the
    whole head and attention query block by query block until `seconds`
    pass (or `max_blocks` blocks are done)."""

    def __init__(self, wl, layer=0):
        import numpy as np
        from cva_workload import chunk_inputs, key_centres, bf16_bits_to_f32
        from oracle import hsa as o_hsa
        from oracle import path as o_path
        self.wl, self.np, self.o_path = wl, np, o_path
        heads = [0]
        centres = key_centres(wl, layer) if wl.keys == "clustered" else None
        self.cache = o_path.FrameCache(wl.B, 1, wl.D, wl.T_f, wl.blk, wl.window)
        self.cache.t_begin = 0
        lo = max(0, wl.t0 + wl.Fc - wl.window)

        def load(c):
            x = chunk_inputs(wl, c, layer, centres=centres)
            return [bf16_bits_to_f32(x[n][:, :, heads]).astype(np.float64) for n in ("q", "k", "v")]

        for c in range(lo // wl.Fc + 1, wl.chunk):
            q, k, v = load(c)
            _, k_rot = o_path.rotate_chunk(q, k, wl.Fh, wl.Fw, wl.Fc, wl.t0_of(c))
            self.cache.append(k_rot, v, wl.t0_of(c), wl.Fc)
        self.q, self.k, self.v = load(wl.chunk)
        self.F = wl.t0 - max(0, wl.t0 + wl.Fc - wl.window)
        self.k_f, self.k_b = o_hsa.budget(wl.chunk, self.F, wl.nb, dense=wl.dense,
                                          k_f_max=wl.k_f_max, d_base=wl.d_base,
                                          d_slope=wl.d_slope, d_pivot=wl.d_pivot,
                                          k_b_fixed=wl.k_b_fixed)

    def run(self, seconds, max_blocks=None):
        np, wl, o_path = self.np, self.wl, self.o_path
        t_start = time.perf_counter()
        run = o_path.run_chunk(self.cache, self.q, self.k, self.v, Fh=wl.Fh, Fw=wl.Fw, Fc=wl.Fc,
                               t0=wl.t0, k_f=self.k_f, k_b=self.k_b, dense=wl.dense,
                               attend_too=False)
        flops = 0.0
        nblk = 0
        tail = wl.T_f - (wl.nb - 1) * wl.blk
        for qb in range(wl.NQB):
            f, j = divmod(qb, wl.nb)
            rows = np.arange(f * wl.T_f + j * wl.blk, f * wl.T_f + min((j + 1) * wl.blk, wl.T_f))
            blocks = run["blocks"]
            o_path.attend_chunk(run["q_rot"], self.cache, wl.t0, wl.Fc, blocks, rows)
            if blocks is None:
                nkeys = self.F * wl.T_f + wl.Lq
            else:
                nkeys = sum(tail if g % wl.nb == wl.nb - 1 else wl.blk for g in blocks[0, 0, qb]) + wl.Lq
            flops += 4.0 * wl.D * len(rows) * nkeys
            nblk += 1
            if time.perf_counter() - t_start > seconds or (max_blocks and nblk >= max_blocks):
                break
        dt = time.perf_counter() - t_start
        desc = (f"fp64 oracle on 1 of {wl.H} heads, {nblk} of {wl.NQB} query blocks "
                f"(rotation, pooling and selection of the whole head included)")
        return flops / dt / 1e12, desc, dt, flops


# ---------------------------------------------------------------- timing

class L2Flush:
    """Evicts L2 between steps: writes 256 MiB, then reads another 256 MiB so
    the cache ends up holding clean lines of neither the flush nor the path."""

    def __init__(self):
        import torch
        self.w = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
        self.r = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device="cuda")

    def zero_(self):
        self.w.zero_()
        self.r.sum()


def time_steps(step, flush, n, stream, stages=True):
    """Runs `step` n times, L2 flushed before each. With `stages`, the
    library's stage events (start, after rotate/append/pool, after
    selection, after attention) are recorded on `stream` and the per-step
    lists in ms are returned: whole step, rotate/append/pool, selection,
    attention. Without, only events around each step are recorded (the
    call then launches its kernels back to back, each allowed to start
    while the previous one drains) and the whole-step list is returned."""
    import torch
    from autoregressive_video_dit_b200 import ops
    st_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4 if stages else 2)] for _ in range(n)]
    for evs in st_ev:
        for e in evs:
            e.record(stream)           # create the underlying events
    torch.cuda.synchronize()
    for i in range(n):
        flush.zero_()
        if stages:
            ops.set_stage_events(st_ev[i])
        else:
            st_ev[i][0].record(stream)
        step()
        if not stages:
            st_ev[i][1].record(stream)
    ops.set_stage_events(None)
    torch.cuda.synchronize()
    if not stages:
        return [e[0].elapsed_time(e[1]) for e in st_ev]
    return ([e[0].elapsed_time(e[3]) for e in st_ev], [e[0].elapsed_time(e[1]) for e in st_ev],
            [e[1].elapsed_time(e[2]) for e in st_ev], [e[2].elapsed_time(e[3]) for e in st_ev])


def rope_kernel_ms(st, rounds=10, sets=4):
    """Per-launch time (ms) of the rotate/append/pool launch alone, through
    its own entry point: `sets` input sets with their own outputs (q_rot,
    pooled queries, and the slots of distinct frames of a scratch cache), in
    total larger than L2, launched back to back round-robin between two
    events on the current stream (each launch reads inputs that three other
    launches' traffic has evicted)."""
    import torch
    from autoregressive_video_dit_b200 import ops
    wl = st["wl"]
    cache = ops.DeviceKVCache(st["shape"], wl.window, 0)
    g = torch.Generator(device="cuda")
    g.manual_seed(1234)
    shp = (wl.B, wl.Lq, wl.H, wl.D)
    sets_ = []
    for i in range(sets):
        q, k, v = (torch.randn(shp, generator=g, device="cuda").to(torch.bfloat16) for _ in range(3))
        q_rot = torch.empty(wl.B * wl.H * wl.Fc * wl.T_pad * wl.D, dtype=torch.bfloat16, device="cuda")
        qpool = torch.empty(wl.B * wl.H * wl.NQB * wl.D, dtype=torch.float32, device="cuda")
        sets_.append((q, k, v, q_rot, qpool, max(0, wl.t0 - wl.Fc * i)))

    def launch(x):
        ops.rotate_append_pool(x[0], x[1], x[2], cache, st["tables"], x[5], x[3], x[4])

    for x in sets_:
        launch(x)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(rounds):
        for x in sets_:
            launch(x)
    e1.record()
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    return e0.elapsed_time(e1) / (rounds * sets)


def reduce_over_ranks(ms, work, device):
    """Weak scaling over independent instances: the job takes as long as its
    slowest rank (max of `ms`) and does the sum of the ranks' `work`. With
    no process group, or one rank, the values pass through."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(ms), float(work)
    t = torch.tensor([float(ms)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    w = torch.tensor([float(work)], device=device, dtype=torch.float64)
    dist.all_reduce(w, op=dist.ReduceOp.SUM)
    return float(t.item()), float(w.item())


def rank_layer(rank):
    """Each rank runs its own instance on the inputs of its own layer seed."""
    return rank


def percentile(xs, q):
    """Nearest-rank percentile (q in [0, 100]) of a non-empty list."""
    ys = sorted(xs)
    k = max(1, math.ceil(q / 100.0 * len(ys)))
    return ys[k - 1]


# ---------------------------------------------------------------- main arms

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from cva_workload import WORKLOADS
    wl = WORKLOADS[args.workload]
    if args.chunk is not None:
        wl = wl.with_chunk(args.chunk)
    n_aff, threads = host_cores()
    times, flops = [], []
    sampler = OracleSample(wl)
    for i in range(args.warmup + args.steps):
        v, desc, dt, fl = sampler.run(0.0, max_blocks=1)
        if i >= args.warmup:
            times.append(dt)
            flops.append(fl)
    value = sum(flops) / sum(times) / 1e12
    ms = 1e3 * statistics.mean(times)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(wl),
        "cpu_baseline": {"kind": "oracle", "value": value, "unit": "TFLOP/s", "cores": threads,
                         "sample": "per step: " + desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(wl):
    return {"workload": f"{wl.key}: {wl.name}", "B": wl.B, "H": wl.H, "D": wl.D,
            "latent_grid": f"{wl.Fh}x{wl.Fw}", "tokens_per_frame": wl.T_f, "chunk_frames": wl.Fc,
            "queries": wl.Lq, "block": wl.blk, "window_frames": wl.window, "chunk_index": wl.chunk,
            "t0": wl.t0, "budget": "dense" if wl.dense else "hierarchical sparse"}


def measure_chunk(args, wl, layer, stream, flush, n, clocks_on, world=1):
    """Times one chunk of `wl` through the fused call: warm-up, then n steps
    with L2 flushed before each, clocks sampled during the timed steps.
    Returns the device state and the per-step stage times (ms)."""
    import torch
    import torch.distributed as dist
    from autoregressive_video_dit_b200 import ops

    st = setup_workload(args, layer=layer, wl=wl)
    wl = st["wl"]

    def step():
        ops.chunk_attention(st["q"], st["k"], st["v"], st["cache"], st["tables"], wl.t0, st["k_f"],
                            st["k_b"], st["ws"], st["out"])

    for _ in range(max(args.warmup, 1)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    flops = attention_flops(st)
    # stage breakdown (a pass of its own, before the timed region)
    staged_ms, rope_ms, sel_ms, attn_ms = time_steps(step, flush, n, stream, stages=True)
    sampler = ClockSampler(enabled=clocks_on)
    time.sleep(0.3 if clocks_on else 0)
    if world > 1:
        dist.barrier()
    step_ms = time_steps(step, flush, n, stream, stages=False)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    assert ops.device_status() == 0
    rope_k = rope_kernel_ms(st)   # after the timed region, on a scratch cache
    return dict(st=st, step=step, flops=flops, step_ms=step_ms, rope_ms=rope_ms, sel_ms=sel_ms,
                attn_ms=attn_ms, staged_ms=staged_ms, rope_kernel_ms=rope_k, clocks=clocks)


def attention_peak(peaks, clocks):
    """The burst bf16 figure for a kernel that ran at full clock; the
    sustained one when the timed region ran into the power cap (a long step)."""
    capped = bool(clocks) and "sw_power_cap" in clocks.get("reasons", [])
    peak = float(peaks["bf16_tflops_sustained" if capped else "bf16_tflops"])
    kind = "bf16 sustained (power cap seen while timing)" if capped else "bf16 burst"
    return peak, kind


def config_entry(m, peaks, peak_src):
    """Per-config summary of one measure_chunk() result."""
    st, wl = m["st"], m["st"]["wl"]
    ms = statistics.mean(m["step_ms"])
    attn = statistics.mean(m["attn_ms"])
    rope = m["rope_kernel_ms"]
    rope_stage = statistics.mean(m["rope_ms"])
    sel = statistics.mean(m["sel_ms"])
    peak, kind = attention_peak(peaks, m["clocks"])
    ach = m["flops"] / (attn * 1e-3) / 1e12
    rb = rope_bytes(wl)
    return {
        "workload": f"{wl.key}: {wl.name}", "chunk_index": wl.chunk, "history_frames": st["F"],
        "k_f": st["k_f"], "k_b": st["k_b"], "budget": "dense" if wl.dense else "hierarchical sparse",
        "ms": ms, "attention_tflop": m["flops"] / 1e12,
        "effective_tflops": m["flops"] / (ms * 1e-3) / 1e12,
        "attention_ms": attn, "attention_tflops": ach,
        "roofline": {"kernel": "attn_fwd_kernel", "bound": "tensor", "achieved": ach, "peak": peak,
                     "unit": "TFLOP/s", "frac": ach / peak,
                     "peak_source": f"{peak_src} {kind}", "flops": "useful: each query block's own keys",
                     "traffic": recorded_traffic("attn_sm100.cu", wl.key)},
        "rotate_append_pool_us": 1e3 * rope,
        "rotate_append_pool_stage_us": 1e3 * rope_stage,
        "roofline_hbm": {"kernel": "rope_pool_tma_kernel", "bound": "hbm",
                         "achieved": rb / (rope * 1e-3) / 1e9, "peak": float(peaks["hbm_gbs"]),
                         "unit": "GB/s", "frac": rb / (rope * 1e-3) / 1e9 / float(peaks["hbm_gbs"]),
                         "algorithmic_bytes": rb,
                         "timing": "per launch of its own entry point, 40 launches back to back over "
                                   "4 input sets larger than L2, CUDA events"},
        "select_us": 1e3 * sel, "select_share": sel / statistics.mean(m["staged_ms"]),
        "ms_stage_pass": statistics.mean(m["staged_ms"]),
        "steps": len(m["step_ms"]), "stat": "mean", "clocks": m["clocks"],
    }


def stream_entry(args, clocks_on, chunks=None):
    """c5 streaming: every chunk through all layers (run_stream's loop),
    per-chunk latency p50/p99 with clocks sampled over the run."""
    sampler = ClockSampler(enabled=clocks_on)
    res = stream_latencies(args, "c5", chunks)
    clocks = sampler.stop()
    res["clocks"] = clocks
    return res


def run_cuda(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    from autoregressive_video_dit_b200 import ops
    from cva_workload import WORKLOADS

    wl = WORKLOADS[args.workload]
    if args.chunk is not None:
        wl = wl.with_chunk(args.chunk)
    stream = torch.cuda.current_stream()
    flush = L2Flush()
    n = args.steps
    m = measure_chunk(args, wl, rank_layer(rank), stream, flush, n, not args.no_clocks, world)
    st, step, flops, clocks = m["st"], m["step"], m["flops"], m["clocks"]
    wl = st["wl"]

    ms = statistics.mean(m["step_ms"])
    ms_max, total_flops = reduce_over_ranks(ms, flops, "cuda")

    # end to end through the public call with pinned host buffers
    e2e = None
    if not args.no_e2e:
        hq = st["q"].cpu().pin_memory()
        hk = st["k"].cpu().pin_memory()
        hv = st["v"].cpu().pin_memory()
        ho = torch.empty(st["out"].shape, dtype=st["out"].dtype).pin_memory()
        ne = min(n, 20)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(ne)]
        for i in range(ne + 2):
            flush.zero_()
            if i >= 2:
                evs[i - 2][0].record(stream)
            st["q"].copy_(hq, non_blocking=True)
            st["k"].copy_(hk, non_blocking=True)
            st["v"].copy_(hv, non_blocking=True)
            step()
            ho.copy_(st["out"], non_blocking=True)
            if i >= 2:
                evs[i - 2][1].record(stream)
        torch.cuda.synchronize()
        e2e_ms, _ = reduce_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in evs), 0.0, "cuda")
        nbytes = lambda t: t.numel() * t.element_size()
        e2e = {"value": total_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": nbytes(hq) + nbytes(hk) + nbytes(hv),
               "d2h_bytes_per_step": nbytes(ho)}

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0

    peaks, peak_src = load_peaks()
    entry = config_entry(m, peaks, peak_src)
    traffic = recorded_traffic("attn_sm100.cu", wl.key)
    line = {
        "metric": METRIC,
        "value": total_flops / (ms_max * 1e-3) / 1e12,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": n,
        "warmup": args.warmup,
        "ms_per_step": ms_max,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) Q/V, keys N(0,1) or clustered; history built through the path)",
        "config": dict(config_of(wl), history_frames=st["F"],
                       k_f=st["k_f"], k_b=st["k_b"], l2="flushed before every step (256 MiB write + 256 MiB read)",
                       parallelism="independent instance per GPU" if world > 1 else "1 GPU"),
        "latency_ms": ms_max,
        "attention_tflop_per_chunk": flops / 1e12,
        "frac_of_bf16_peak": (total_flops / world) / (ms_max * 1e-3) / 1e12 / entry["roofline"]["peak"],
        "stage_ms": {"rotate_append_pool": entry["rotate_append_pool_stage_us"] * 1e-3,
                     "select": entry["select_us"] * 1e-3, "attention": entry["attention_ms"],
                     "step_with_stage_events": entry["ms_stage_pass"],
                     "note": "a separate pass with events between the stages (kernels then launch "
                             "one after another); latency_ms is the timed pass without them"},
        "roofline": dict(entry["roofline"], traffic=traffic),
        "roofline_hbm": entry["roofline_hbm"],
        "gpu_launches": n * launches_per_step(wl, st),
        "clocks": clocks,
    }
    if e2e:
        line["e2e"] = e2e
    if world == 1 and not args.no_per_config:
        per = {}
        for key, chunk in (("c2", None), ("c3", 7)):
            if key == wl.key and (chunk is None or chunk == wl.chunk):
                continue
            w2 = WORKLOADS[key] if chunk is None else WORKLOADS[key].with_chunk(chunk)
            m2 = measure_chunk(args, w2, 0, stream, flush, n, not args.no_clocks)
            per[key] = config_entry(m2, peaks, peak_src)
            del m2
            torch.cuda.empty_cache()
        per["c5"] = stream_entry(args, not args.no_clocks)
        line["per_config"] = per
    if world == 1 and not args.no_cpu_baseline:
        n_aff, threads = host_cores()
        v, desc, dt, _ = OracleSample(wl).run(args.cpu_seconds)
        desc += f", {dt:.1f} s"
        line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                "sample": desc}
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def launches_per_step(wl, st):
    """Kernel launches of one fused chunk call: rotate/append/pool; the
    selection (sparse budget with history) and the query-block pairing (64-row
    blocks, a history of at least 2 k_f frames); the attention, plus the merge
    of split tail tiles."""
    sparse = st["k_f"] >= 0 and st["F"] > 0
    n = 1 + attention_launches(wl)
    if sparse:
        n += 1 + int(wl.blk == 64 and st["F"] >= 2 * min(st["k_f"], st["F"]))
    return n


def run_sweep(args):
    """Per-chunk cost under the density schedule and its mirror (chunk 1 is
    dense: no history)."""
    import torch
    from autoregressive_video_dit_b200 import ops
    from cva_workload import WORKLOADS
    base = WORKLOADS[args.workload]
    stream = torch.cuda.current_stream()
    flush = L2Flush()
    # third schedule: density from the noise level (s_base 0.8, target 0.75)
    noise = ops.cag_noise_densities(base.chunks, base.Fc, base.window, base.nb, 0.8, 0.75)
    # fourth: the top-p budget (p = 0.9, capped at every candidate block)
    schedules = [("literal", base.d_slope, None, None), ("mirrored", -base.d_slope, None, None),
                 ("noise s_base=0.8 s_target=0.75", base.d_slope, noise, None),
                 ("top-p p=0.9", base.d_slope, None, 0.9)]
    for sched, slope, dens, topp in schedules:
        for chunk in range(1, base.chunks + 1):
            wl = base.replace(d_slope=slope).with_chunk(chunk)
            hist = min(base.Fc * (chunk - 1), base.window - base.Fc)
            if dens is not None and chunk >= 2:
                _, kb = ops.cag_density_budget(chunk, hist, base.nb, base.k_f_max, dens[chunk])
                wl = wl.replace(k_b_fixed=kb)
            if topp is not None and chunk >= 2:
                wl = wl.replace(k_b_fixed=min(base.k_f_max, hist) * base.nb)   # the cap
            st = setup_workload(args, layer=0, wl=wl)
            use_topp = topp is not None and st["F"] > 0

            def step():
                if use_topp:
                    ops.chunk_attention_topp(st["q"], st["k"], st["v"], st["cache"], st["tables"], wl.t0,
                                             st["k_f"], st["k_b"], topp, st["ws"], st["out"])
                else:
                    ops.chunk_attention(st["q"], st["k"], st["v"], st["cache"], st["tables"], wl.t0,
                                        st["k_f"], st["k_b"], st["ws"], st["out"])

            for _ in range(max(args.warmup, 1)):
                flush.zero_()
                step()
            torch.cuda.synchronize()
            assert ops.device_status() == 0
            flops = attention_flops(st)
            mean_blocks = st["k_b"]
            if use_topp:
                mean_blocks = float(block_lists(st)[1].mean())
            step_ms, rope_ms, sel_ms, attn_ms = time_steps(step, flush, args.steps, stream)
            assert ops.device_status() == 0
            ms = statistics.median(step_ms)
            print(json.dumps({
                "mode": "schedule sweep", "workload": wl.key, "schedule": sched, "chunk": chunk,
                "history_frames": st["F"], "k_f": st["k_f"], "k_b": st["k_b"],
                "mean_blocks": mean_blocks,
                "ms": ms, "attention_ms": statistics.median(attn_ms),
                "select_us": 1e3 * statistics.median(sel_ms),
                "select_share": statistics.median(sel_ms) / ms,
                "rotate_append_pool_us": 1e3 * statistics.median(rope_ms),
                "attention_tflop": flops / 1e12,
                "attention_tflops": flops / (statistics.median(attn_ms) * 1e-3) / 1e12,
                "steps": args.steps, "stat": "median"}), flush=True)
            del st
    return 0


def stream_latencies(args, key, chunks=None):
    """Every chunk of the workload once (or the first `chunks`), through all
    its layers, each layer with its own cache (rolling window); per-chunk
    latency = the sum over layers, timed from the first layer's start to the
    last layer's end. Inputs are drawn on the device from a seeded generator
    per (chunk, layer), outside the timed region."""
    import torch
    from autoregressive_video_dit_b200 import ops
    from cva_workload import WORKLOADS
    wl = WORKLOADS[key]
    nch = wl.chunks if chunks is None else chunks
    shape = ops.make_shape(wl.B, wl.H, wl.D, wl.Fh, wl.Fw, wl.Fc, wl.blk)
    tables = ops.DeviceRopeTables(wl.D, wl.Fc * wl.chunks, wl.Fh, wl.Fw)
    caches = [ops.DeviceKVCache(shape, wl.window, 0) for _ in range(wl.layers)]
    budgets = []
    for c in range(1, wl.chunks + 1):
        hist = min(wl.Fc * (c - 1), wl.window - wl.Fc)
        budgets.append(ops.cag_budget(c, hist, wl.nb, dense=wl.dense, k_f_max=wl.k_f_max,
                                      d_base=(wl.d_base.numerator, wl.d_base.denominator),
                                      d_slope=(wl.d_slope.numerator, wl.d_slope.denominator),
                                      pivot=wl.d_pivot, k_b_fixed=wl.k_b_fixed) if hist > 0 else (0, 0))
    k_f_max = max(b[0] for b in budgets)
    k_b_max = max(b[1] for b in budgets)
    ws = torch.empty(ops.chunk_workspace_bytes(shape, k_f_max, k_b_max), dtype=torch.uint8, device="cuda")
    out = torch.empty((wl.B, wl.Lq, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    gen = torch.Generator(device="cuda")
    size = (wl.B, wl.Lq, wl.H, wl.D)

    def inputs(c, layer):
        gen.manual_seed(1_000_000 * wl.config_index + 1_000 * c + layer)
        return [torch.randn(size, generator=gen, device="cuda").to(torch.bfloat16) for _ in range(3)]

    def run_chunk(c, timed):
        k_f, k_b = budgets[c - 1]
        t0 = wl.t0_of(c)
        xs = [inputs(c, layer) for layer in range(wl.layers)]
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for layer in range(wl.layers):
            q, k, v = xs[layer]
            ops.chunk_attention(q, k, v, caches[layer], tables, t0, k_f, k_b, ws, out)
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) if timed else None

    for c in (1, 2):                      # warm-up, then the caches start over
        run_chunk(c, False)
    caches = [ops.DeviceKVCache(shape, wl.window, 0, arena=x.arena) for x in caches]
    lat = [run_chunk(c, True) for c in range(1, nch + 1)]
    assert ops.device_status() == 0
    full = wl.window // wl.Fc + 1          # first chunk whose history fills the window
    steady = lat[full - 1:]
    res = {
        "mode": "streaming", "workload": f"{wl.key}: {wl.name}", "chunks": nch, "layers": wl.layers,
        "window_frames": wl.window, "unit": "ms per chunk (all layers)",
        "p50": percentile(lat, 50), "p99": percentile(lat, 99), "max": max(lat),
        "chunk1": lat[0], "steady_p50": percentile(steady, 50) if steady else None,
        "steady_from_chunk": full,
        "budget_first_full_window": {"k_f": budgets[full - 1][0], "k_b": budgets[full - 1][1]},
        "per_chunk": [round(x, 3) for x in lat]}
    del caches, ws, out
    torch.cuda.empty_cache()
    return res


def run_stream(args):
    print(json.dumps(stream_latencies(args, args.workload)), flush=True)
    return 0


def run_qkv(args):
    """Fused QKV projection + rotation + append + pooling of one chunk, against
    the unfused route on the same inputs: three cuBLAS GEMMs (q, k, v), then
    cva_rope3d_apply + cva_hsa_compress for q and cva_kv_append for k, v.
    Medians of --steps runs, L2 flushed before each."""
    import numpy as np
    import torch
    from autoregressive_video_dit_b200 import ops
    from cva_workload import WORKLOADS, hidden_inputs
    wl = WORKLOADS[args.workload]
    C = wl.H * wl.D
    inp = hidden_inputs(wl, C)
    dev = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)
    x, w = dev(inp["x"]), dev(inp["w"])
    shape = ops.make_shape(wl.B, wl.H, wl.D, wl.Fh, wl.Fw, wl.Fc, wl.blk)
    tables = ops.DeviceRopeTables(wl.D, wl.t0 + wl.Fc, wl.Fh, wl.Fw)
    cache = ops.DeviceKVCache(shape, wl.window, 0)
    q_rot = torch.empty((wl.B, wl.H, wl.Fc * wl.T_pad, wl.D), dtype=torch.bfloat16, device="cuda")
    qpool = torch.empty((wl.B, wl.H, wl.NQB, wl.D), dtype=torch.float32, device="cuda")
    HD = wl.H * wl.D
    wq, wk, wv = w[:HD], w[HD:2 * HD], w[2 * HD:]
    flush = L2Flush()

    def fused():
        ops.qkv_rope_append(x, w, cache, tables, wl.t0, q_rot, qpool)

    def unfused():
        q = torch.matmul(x, wq.t())
        k = torch.matmul(x, wk.t())
        v = torch.matmul(x, wv.t())
        ops.rope3d_apply(q, q_rot, tables, shape, wl.t0, 1)
        ops.hsa_compress(q_rot, shape, qpool)
        ops.kv_append(k, v, cache, tables, wl.t0)

    def timed(fn):
        for _ in range(max(args.warmup, 1)):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        ms = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        return statistics.median(ms)

    f_ms = timed(fused)
    u_ms = timed(unfused)
    assert ops.device_status() == 0
    flops = 2.0 * wl.B * wl.Lq * C * 3 * HD
    peaks, src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    print(json.dumps({
        "mode": "qkv projection", "workload": wl.key, "hidden": C, "gemm": f"[{wl.B * wl.Lq} x {C}] x [{C} x {3 * HD}]",
        "fused_us": 1e3 * f_ms, "fused_tflops": flops / (f_ms * 1e-3) / 1e12,
        "fused_frac_of_bf16_peak": flops / (f_ms * 1e-3) / 1e12 / peak, "peak_source": f"{src} bf16 burst",
        "unfused_us": 1e3 * u_ms, "speedup": u_ms / f_ms, "steps": args.steps, "stat": "median",
        "launches": {"fused": 2, "unfused": 3 + 4}}), flush=True)
    return 0


def run_mma_shapes(args):
    """Cycles per back-to-back tcgen05.mma (bf16, K = 16) for the tile shapes the
    attention could use, one CTA per SM; the median over the SMs of the
    second of two runs."""
    import torch
    from autoregressive_video_dit_b200 import ops
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cycles = torch.zeros(sms, dtype=torch.int64, device="cuda")
    iters = 1024
    for m, n in ((128, 128), (64, 128), (128, 256), (64, 256), (128, 64), (64, 64)):
        for _ in range(2):
            ops.diag_mma_cycles(m, n, iters, cycles)
            torch.cuda.synchronize()
        assert ops.device_status() == 0
        per = float(cycles.median().item()) / (4 * iters)
        print(json.dumps({"mode": "mma shapes", "m": m, "n": n, "k": 16, "cycles_per_mma": per,
                          "flop_per_cycle_per_sm": 2.0 * m * n * 16 / per, "ctas": sms,
                          "mmas_per_cta": 4 * iters}), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.qkv:
        return run_qkv(args)
    if args.sweep:
        return run_sweep(args)
    if args.stream:
        return run_stream(args)
    if args.mma_shapes:
        return run_mma_shapes(args)
    return run_cuda(args)


if __name__ == "__main__":
    sys.exit(main())
