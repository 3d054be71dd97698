"""fp64 CPU oracle of the per-chunk attention path (TEST INFRASTRUCTURE).

This package is a plain, slow, obviously correct restatement of what the
CUDA library computes. It exists so the tests, the smoke check and the
bench's CPU baseline have something independent to compare against. It
shares no code with ``autoregressive_video_dit_b200`` (neither imports the
other) and no product code path may call it: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg use it.

Sources (the method as the pages describe it):

* "Accelerating Video Generation Inference with Sequential-Parallel 3D
  Positional Encoding Using a Global Time Index" (Causal-RoPE SP),
  technical summary section 2B: every chunk carries a start-frame offset
  ``s`` and a token at local frame ``t`` takes the global time index
  ``t + s``; section 2C: cos/sin frequencies are precomputed into
  contiguous tables.
* "Light Forcing", section 2.1 (Chunk-Aware Growth: the first chunk is
  dense, the budget per chunk is a schedule) and section 2.2 (Hierarchical
  Sparse Attention: mean-pool Q and K per block and per frame, pick frames
  per query block from frame-pooled keys, then blocks inside the picked
  frames from block-pooled keys, then attend only to the picked
  frame-block pairs).

Modules:

* :mod:`oracle.rope`      -- 3D rotary embedding with a global time index.
* :mod:`oracle.hsa`       -- pooling, two-level top-k selection, budgets.
* :mod:`oracle.attention` -- chunk attention over an explicit key set.
* :mod:`oracle.path`      -- a frame cache and the whole per-chunk path.
* :mod:`oracle.qkv`       -- QKV projection followed by Causal-RoPE.

Where the pages leave a step open the oracle takes one reading, named in
each function's docstring. Functions whose behaviour rests on such a
reading only (no value, law or special case on the pages fixes it) say
"parity unpinned" in their docstring: ``axis_split`` (how head_dim is
shared among t/h/w), ``frame_select``'s choice of the block-pooled query
as the frame-selection query, and ``budget``'s density schedule direction.
"""

from . import rope, hsa, attention, path  # noqa: F401

__all__ = ["rope", "hsa", "attention", "path"]
