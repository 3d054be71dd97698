"""The fused chunk call for callers that cannot allocate device memory.

A plugin whose host runtime owns every allocation and hands it only its
inputs and outputs, or a loop that may not allocate after start-up, cannot
pass a workspace. cva_chunk_attention_noalloc serves such callers from a
fixed scratch array inside the library. These tests call it through the C
ABI and check that it reproduces cva_chunk_attention with a caller
workspace bit for bit (both run the same kernels on the same inputs), on
two calls in a row; that after its first call further calls allocate no
device memory; and that a shape needing more scratch than the array holds
is refused before anything runs, while a bad budget is refused as such.
"""
import numpy as np
import pytest

from cva_workload import WORKLOADS, key_centres
from _util import from_dev, inputs, lib_budget, shape_of, to_dev

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
    # the chunk's own frames are rewritten by every call with the same values,
    # so the calls below all see the same cache
    ws = torch.empty(ops.chunk_workspace_bytes(shp, k_f, k_b), dtype=torch.uint8, device="cuda")
    ref = torch.empty((wl.B, wl.Lq, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    ops.chunk_attention(q, k, v, cache, tabs, t0, k_f, k_b, ws, ref)
    torch.cuda.synchronize()
    want = from_dev(ref)

    outs = [torch.full_like(ref, float("nan")) for _ in range(2)]
    ops.chunk_attention_noalloc(q, k, v, cache, tabs, t0, k_f, k_b, outs[0])   # first call: set-up
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    stats0 = torch.cuda.memory_stats()
    ops.chunk_attention_noalloc(q, k, v, cache, tabs, t0, k_f, k_b, outs[1])
    torch.cuda.synchronize()
    # the second call allocated nothing on the device
    assert torch.cuda.mem_get_info()[0] == free0
    stats1 = torch.cuda.memory_stats()
    for key_ in ("allocation.all.allocated", "segment.all.allocated"):
        assert stats1.get(key_, 0) == stats0.get(key_, 0), key_
    for call, out in enumerate(outs):
        np.testing.assert_array_equal(from_dev(out), want, err_msg=f"call {call}")
    assert ops.device_status() == 0


def _c4_buffers():
    """Real device buffers of the 14B 720P chunk (cache, tables, q, k, v, out)."""
    import torch
    from autoregressive_video_dit_b200 import ops
    wl = WORKLOADS["c4"]
    shp = shape_of(wl)
    cache = ops.DeviceKVCache(shp, wl.window)
    tabs = ops.DeviceRopeTables(wl.D, wl.t0 + wl.Fc, wl.Fh, wl.Fw)
    q, k, v, out = (torch.zeros((wl.B, wl.Lq, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
                    for _ in range(4))
    return wl, cache, tabs, q, k, v, out


def test_noalloc_refuses_a_shape_beyond_its_scratch():
    import torch
    from autoregressive_video_dit_b200 import ops

    wl, cache, tabs, q, k, v, out = _c4_buffers()   # ~115 MB of scratch needed
    k_f, k_b = lib_budget(wl, wl.chunk)
    with pytest.raises(ops.CvaError) as e:
        ops.chunk_attention_noalloc(q, k, v, cache, tabs, wl.t0, k_f, k_b, out)
    assert e.value.code == ops.CVA_ENOMEM
    assert "scratch" in ops.last_error()
    # a budget beyond the candidates is a range error, whatever the scratch
    with pytest.raises(ops.CvaError) as e:
        ops.chunk_attention_noalloc(q, k, v, cache, tabs, wl.t0, k_f, k_f * wl.nb + 1, out)
    assert e.value.code == ops.CVA_ERANGE
    torch.cuda.synchronize()
    assert ops.device_status() == 0
