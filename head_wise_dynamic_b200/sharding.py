"""Head-sharded execution over several GPUs (one process per GPU, torch.distributed).

The 16 heads of a global-attention layer are independent: each has its own kept
sets, its own index cache and its own output rows.  Rank r of G takes the
contiguous heads [r*H/G, (r+1)*H/G) of Q/K/V ([H][N][64], so a rank's heads are
one contiguous slice), builds and caches only their index sets (the DINO tile
ranking is recomputed per rank: it is per input and cheap), runs the sparse
attention on them, and - when the consumer of O is not head-sharded - one
all-gather over NCCL (NVLink / NVSwitch) assembles O on every rank.  There is no
collective inside the attention itself.

This module is plumbing around the library: the partition of the heads and the
collective.  Every step of the attention runs in the library's kernels.
"""
from __future__ import annotations

from typing import Sequence, Tuple

from . import SparseGlobalAttention


def head_range(H: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous heads [h0, h1) of `rank` among `world` ranks; H must divide evenly so that
    every rank's output block has the same shape (the all-gather needs it)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank out of range")
    if H % world:
        raise ValueError(f"{H} heads do not split evenly over {world} ranks")
    per = H // world
    return rank * per, (rank + 1) * per


def gather_heads(local_out, full_out, group=None):
    """All-gather the ranks' [H/G][N][64] output blocks into full_out [H][N][64] (rank order =
    head order).  NCCL gathers straight into the output; other backends use a list gather."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        full_out.copy_(local_out)
        return full_out
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(full_out, local_out.contiguous(), group=group)
    else:
        parts = list(torch.chunk(full_out, dist.get_world_size(group), dim=0))
        dist.all_gather(parts, local_out.contiguous(), group=group)
    return full_out


class ShardedGlobalAttention:
    """The heads of this rank (see head_range) with their own index cache and workspace.

    select() and __call__() take the full [H][N][64] tensors and use this rank's slice;
    __call__ returns the full output (gathered) or, with gather=False, the local block."""

    def __init__(self, layout, heads: Sequence, world: int = 1, rank: int = 0, device="cuda", out_dtype=None,
                 group=None):
        self.H = len(heads)
        self.h0, self.h1 = head_range(self.H, world, rank)
        self.group = group
        self.local_heads = list(heads[self.h0:self.h1])
        self.layout = _sub_layout(layout, self.h1 - self.h0)
        self.att = SparseGlobalAttention(self.layout, self.local_heads, device=device, out_dtype=out_dtype)
        self.full_out = None

    def _mine(self, t):
        return t[self.h0:self.h1]

    def select(self, q, k, dino=None, stream=None):
        self.att.select(self._mine(q), self._mine(k), dino, stream)

    def __call__(self, q, k, v, out=None, gather: bool = True, stream=None):
        local = self.att(self._mine(q), self._mine(k), self._mine(v), stream=stream)
        if not gather:
            return local
        if out is None:
            if self.full_out is None:
                import torch
                self.full_out = torch.empty((self.H,) + tuple(local.shape[1:]), dtype=local.dtype,
                                            device=local.device)
            out = self.full_out
        return gather_heads(local, out, self.group)


def _sub_layout(layout, H: int):
    """A copy of `layout` (a synthetic Layout or a saf3r_layout) with H heads."""
    from . import saf3r_layout
    if isinstance(layout, saf3r_layout):
        sub = saf3r_layout()
        for name, _ in saf3r_layout._fields_:
            setattr(sub, name, getattr(layout, name))
        sub.H = H
        return sub
    import dataclasses
    if dataclasses.is_dataclass(layout):
        return dataclasses.replace(layout, H=H)
    raise TypeError("layout must be a saf3r_layout or a dataclass layout")
