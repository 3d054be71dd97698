"""Per-chunk attention path of a causal autoregressive video DiT on B200.

The work runs in ``libcva.so`` (hand-written sm_100a CUDA behind the C ABI of
``include/cva.h``); this package only marshals torch tensors into it.
Build the library with ``python -m autoregressive_video_dit_b200.build``.

``from autoregressive_video_dit_b200 import ops`` loads the library (and
raises if it is not built); importing the package itself does not.
"""

__all__ = ["ops", "lib_path"]


def lib_path() -> str:
    import os
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcva.so")


def __getattr__(name):
    if name == "ops":
        from . import _native
        return _native
    raise AttributeError(name)
