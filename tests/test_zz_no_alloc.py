"""The fused chunk call for callers that cannot allocate device memory.

A plugin whose host runtime owns every allocation and hands it only its
inputs and outputs, or a loop that may not allocate after start-up, cannot
pass a workspace. cva_chunk_attention_noalloc serves such callers from a
fixed scratch array inside the library. These tests call it through the C
ABI and check that it reproduces cva_chunk_attention with a caller
workspace, on two calls in a row, and that a shape needing more scratch
than the array holds is refused before anything runs.
"""
import ctypes

import numpy as np
import pytest

from cva_workload import WORKLOADS, key_centres
from _util import MAX_ABS, MEAN_ABS, bits_to_f64, from_dev, inputs, lib_budget, shape_of, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("key,chunk", [("r64", 3), ("c3", 4)])
def test_noalloc_matches_the_workspace_call(key, chunk):
    import torch
    from autoregressive_video_dit_b200 import ops

    wl = WORKLOADS[key]
    shp = shape_of(wl)
    tabs = ops.DeviceRopeTables(wl.D, wl.t0_of(chunk) + wl.Fc, wl.Fh, wl.Fw)
    cache = ops.DeviceKVCache(shp, wl.window)
    centres = key_centres(wl, 0) if wl.keys == "clustered" else None
    for c in range(1, chunk):
        x = inputs(wl, c, 0, None, centres)
        ops.kv_append(to_dev(x["k"]), to_dev(x["v"]), cache, tabs, wl.t0_of(c))
    x = inputs(wl, chunk, 0, None, centres)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    t0 = wl.t0_of(chunk)
    k_f, k_b = lib_budget(wl, chunk)
    assert k_b > 0

    ws = torch.empty(ops.chunk_workspace_bytes(shp, k_f, k_b), dtype=torch.uint8, device="cuda")
    ref = torch.empty((wl.B, wl.Lq, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    ops.chunk_attention(q, k, v, cache, tabs, t0, k_f, k_b, ws, ref)
    torch.cuda.synchronize()
    want = bits_to_f64(from_dev(ref))

    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        ops.chunk_attention_noalloc(q, k, v, cache, tabs, t0, k_f, k_b, out)
        torch.cuda.synchronize()
        got = bits_to_f64(from_dev(out))
        assert np.isfinite(got).all(), call
        d = np.abs(got - want)
        assert d.max() <= MAX_ABS and d.mean() <= MEAN_ABS, (call, d.max(), d.mean())
    assert ops.device_status() == 0


def test_noalloc_refuses_a_shape_beyond_its_scratch():
    from autoregressive_video_dit_b200 import ops

    wl = WORKLOADS["c4"]        # 14B 720P chunk: ~115 MB of scratch
    shp = shape_of(wl)
    cache = ops.KVCache()
    nbytes = ops.kv_cache_bytes(shp, wl.window)
    # the arena is never touched: the size check runs first
    assert ops.lib.cva_kv_cache_init(ctypes.byref(cache), ctypes.c_void_p(1 << 40), nbytes,
                                     ctypes.byref(shp), wl.window, 0) == ops.CVA_OK
    tabs = ops.RopeTables()
    fake = ctypes.c_void_p(1 << 41)
    rc = ops.lib.cva_chunk_attention_noalloc(fake, fake, fake, ctypes.byref(cache), ctypes.byref(tabs),
                                             18, 6, 104, fake, None, None)
    assert rc == ops.CVA_ENOMEM
    assert "scratch" in ops.last_error()
