"""Head-sharded chunk attention across ranks (one process per GPU).

"Accelerating Video Generation Inference with Sequential-Parallel 3D
Positional Encoding Using a Global Time Index": section 2A splits the
chunk's tokens across P ranks (sequence parallelism); section 2C replaces
the separate exchanges of Q, K and V by one fused all-to-all. Here one
all-to-all carries Q, K and V together and hands every rank all tokens of
H/P heads; the rank runs the whole per-chunk path on its heads against its
own frame cache (the rotation needs only the global time index, section 2B);
a second all-to-all returns the output's token slices.

The layout steps around the exchanges run in the library
(``cva_copy_rows_2d``); the exchanges are ``torch.distributed`` all-to-alls
(NCCL between GPUs). ``ShardPlan`` holds the byte plans of those copies so
that they can be checked without a GPU.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional


@dataclass(frozen=True)
class ShardPlan:
    """Sizes of one rank's exchange for a chunk of ``Lq`` tokens of ``H``
    heads of ``D`` elements over ``P`` ranks (element size ``esz`` bytes).
    Every copy is ``(n0, n1, inner, (ss0, ss1), (ds0, ds1), src_off, dst_off)``
    in bytes, for :func:`autoregressive_video_dit_b200.ops.copy_rows_2d`."""
    B: int
    Lq: int
    H: int
    D: int
    P: int
    esz: int = 2

    def __post_init__(self):
        if self.P < 1 or self.H % self.P or self.Lq % self.P:
            raise ValueError(f"heads {self.H} and tokens {self.Lq} must split evenly over {self.P} ranks")
        if (self.H // self.P * self.D * self.esz) % 16:
            raise ValueError("a rank's head group must span a multiple of 16 bytes")

    @property
    def L(self) -> int:          # tokens per rank
        return self.Lq // self.P

    @property
    def Hl(self) -> int:         # heads per rank
        return self.H // self.P

    @property
    def row(self) -> int:        # bytes of one token's head group
        return self.Hl * self.D * self.esz

    @property
    def slab(self) -> int:       # bytes of one tensor's token slice for one head group
        return self.B * self.L * self.row

    def pack(self, t: int):
        """Token slice [B][L][P][row] of tensor t -> send [P][3][B][L][row]."""
        B, L, P, row = self.B, self.L, self.P, self.row
        return (B * L, P, row, (P * row, row), (row, 3 * self.slab), 0, t * self.slab)

    def unpack(self, t: int):
        """recv [P][3][B][L][row] -> tensor t of the rank's heads [B][P*L][row]."""
        B, L, P, row = self.B, self.L, self.P, self.row
        return (P, B, L * row, (3 * self.slab, L * row), (L * row, P * L * row), t * self.slab, 0)

    def pack_out(self):
        """Output of the rank's heads [B][P*L][row] -> send [P][B][L][row]."""
        B, L, P, row = self.B, self.L, self.P, self.row
        return (B, P, L * row, (P * L * row, L * row), (L * row, B * L * row), 0, 0)

    def unpack_out(self):
        """recv [P][B][L][row] (head group g from rank g) -> output slice [B][L][P][row]."""
        B, L, P, row = self.B, self.L, self.P, self.row
        return (P, B * L, row, (B * L * row, row), (row, P * row), 0, 0)


def _apply(copy_rows, src, dst, spec):
    """Runs one copy of a plan on flat byte views of src and dst."""
    import torch
    n0, n1, inner, ss, ds, so, do = spec
    copy_rows(src.reshape(-1).view(torch.uint8)[so:], dst.reshape(-1).view(torch.uint8)[do:], n0, n1, inner, ss, ds)


class HeadShardedChunkAttention:
    """The per-chunk path with the chunk sharded by tokens across the ranks of
    ``group`` and the work sharded by heads.

    Each rank passes its token slice ``q, k, v`` ``[B, Lq/P, H, D]`` (bf16) and
    gets the attention output of the same tokens, all heads, in ``out``
    (contiguous). The rank's frame cache holds its H/P heads. A call is three
    phases around the two exchanges (``pack``, ``compute``, ``finish``);
    ``rank`` and ``world`` may be given instead of a process group to drive
    the phases of several ranks from one process. ``copy_rows`` and
    ``attend`` default to the library; tests substitute host versions.
    """

    def __init__(self, shape, window: int, tables, group=None, t_begin: int = 0, device="cuda",
                 copy_rows: Optional[Callable] = None, attend: Optional[Callable] = None,
                 rank: Optional[int] = None, world: Optional[int] = None):
        from . import _native as ops
        if rank is None or world is None:
            import torch.distributed as dist
            rank, world = dist.get_rank(group), dist.get_world_size(group)
        self.group = group
        self.P = world
        self.rank = rank
        self.shape = shape
        dd = ops.dims(shape)
        self.plan = ShardPlan(shape.batch, dd["Lq"], shape.heads, shape.head_dim, self.P)
        self.local_shape = ops.make_shape(shape.batch, self.plan.Hl, shape.head_dim, shape.frame_h,
                                          shape.frame_w, shape.chunk_frames, shape.block)
        self.tables = tables
        self.device = device
        self.copy_rows = copy_rows or ops.copy_rows_2d
        if attend is None:
            self.cache = ops.DeviceKVCache(self.local_shape, window, t_begin, device=device)
            attend = self._attend_native
        self.attend = attend
        # Buffers kept across calls (allocated on first use): the exchange
        # buffers, the rank's whole-chunk Q, K, V and output of its heads, and
        # the chunk workspace (grown when a larger budget needs more).
        self._bufs = {}
        self.ws = None

    def _buf(self, name, numel, dtype, device):
        import torch
        t = self._bufs.get(name)
        if t is None or t.numel() != numel or t.dtype != dtype or t.device != torch.device(device):
            t = torch.empty(numel, dtype=dtype, device=device)
            self._bufs[name] = t
        return t

    def _attend_native(self, q, k, v, t0, k_f, k_b, out):
        import torch
        from . import _native as ops
        need = ops.chunk_workspace_bytes(self.local_shape, k_f, k_b)
        if self.ws is None or self.ws.numel() < need or self.ws.device != q.device:
            self.ws = torch.empty(need, dtype=torch.uint8, device=q.device)
        ops.chunk_attention(q, k, v, self.cache, self.tables, t0, k_f, k_b, self.ws, out)

    def pack(self, q, k, v):
        """The rank's token slices of Q, K and V laid out for the exchange: [P][3][B][L][row]."""
        pl = self.plan
        send = self._buf("send", 3 * pl.slab * pl.P // q.element_size(), q.dtype, q.device)
        for t, x in enumerate((q, k, v)):
            _apply(self.copy_rows, x.contiguous(), send, pl.pack(t))
        return send

    def compute(self, recv, t0: int, k_f: int, k_b: int):
        """The path on this rank's heads from the exchanged Q, K and V; returns
        the output laid out for the exchange back: [P][B][L][row]."""
        pl = self.plan
        B, Hl, D = pl.B, pl.Hl, pl.D
        n = B * pl.Lq * Hl * D
        loc = [self._buf(f"loc{t}", n, recv.dtype, recv.device).view(B, pl.Lq, Hl, D) for t in range(3)]
        for t in range(3):
            _apply(self.copy_rows, recv, loc[t], pl.unpack(t))
        out_l = self._buf("out_l", n, recv.dtype, recv.device).view(B, pl.Lq, Hl, D)
        self.attend(loc[0], loc[1], loc[2], t0, k_f, k_b, out_l)
        send2 = self._buf("send2", pl.slab * pl.P // recv.element_size(), recv.dtype, recv.device)
        _apply(self.copy_rows, out_l, send2, pl.pack_out())
        return send2

    def finish(self, recv2, out) -> None:
        """Every head group's output for this rank's tokens into ``out`` [B, L, H, D]."""
        if not out.is_contiguous():
            raise ValueError("out must be contiguous")
        _apply(self.copy_rows, recv2, out, self.plan.unpack_out())

    def __call__(self, q, k, v, t0: int, k_f: int, k_b: int, out) -> None:
        import torch.distributed as dist
        send = self.pack(q, k, v)
        recv = self._buf("recv", send.numel(), send.dtype, send.device)
        dist.all_to_all_single(recv, send, group=self.group)     # one exchange for Q, K and V
        send2 = self.compute(recv, t0, k_f, k_b)
        recv2 = self._buf("recv2", send2.numel(), send2.dtype, send2.device)
        dist.all_to_all_single(recv2, send2, group=self.group)
        self.finish(recv2, out)
