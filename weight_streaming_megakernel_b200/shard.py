"""Column-parallel (N-split) decode GEMMs across ranks.

Each of `world` ranks holds the rows W[n0:n1, :] of every weight -- a
contiguous block of output columns -- and a replica of X; it computes its
block Y[:, n0:n1] and, where the consumer needs all of Y, one all-gather
assembles the full [M, N] on every rank.  The weight bytes each GPU streams
shrink by `world`; the exchange is M * N * 2 bytes per GEMM (786 KB for the
Qwen3-8B gate+up projection at M = 16), small next to the streamed weights.

Block boundaries are multiples of `align` output columns: the weight tile
height of the kernel path (128 rows on the tensor-core path, 16 or 32 on the
FMA path), and 16 for the fused SiLU*mul weight, whose gate/up pairs come in
blocks of 16 rows (8 output columns).

This module is host logic around the library: `ShardedLinear` calls the
library's GEMM (or, in CPU tests of the sharding itself, any function with
the same contract) and torch.distributed's all-gather.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch


def column_shards(N: int, world: int, align: int = 128) -> List[Tuple[int, int]]:
    """Contiguous [n0, n1) blocks of N output columns for `world` ranks:
    boundaries are multiples of `align`, the blocks differ by at most one
    `align` unit, and the last block takes the ragged remainder.  A rank may
    get an empty block when N has fewer than `world` units."""
    if N < 0 or world < 1 or align < 1:
        raise ValueError("need N >= 0, world >= 1, align >= 1")
    units = -(-N // align)
    base, extra = divmod(units, world)
    out, u = [], 0
    for r in range(world):
        cnt = base + (1 if r < extra else 0)
        n0 = min(N, u * align)
        n1 = min(N, (u + cnt) * align)
        out.append((n0, n1))
        u += cnt
    return out


def shard_rows(w: torch.Tensor, rank: int, world: int, align: int = 128) -> torch.Tensor:
    """This rank's rows of a weight [N, K] (a contiguous copy)."""
    n0, n1 = column_shards(w.shape[0], world, align)[rank]
    return w[n0:n1].contiguous()


def gather_columns(y_shard: torch.Tensor, shards: Sequence[Tuple[int, int]], group=None) -> torch.Tensor:
    """All-gather the ranks' column blocks into the full [M, N] on every rank.
    Blocks are padded to the widest one so one all_gather_into_tensor moves
    them all; the padding is dropped when the full matrix is assembled."""
    import torch.distributed as dist

    world = len(shards)
    M = y_shard.shape[0]
    widest = max(n1 - n0 for n0, n1 in shards)
    send = torch.zeros(M, widest, dtype=y_shard.dtype, device=y_shard.device)
    send[:, : y_shard.shape[1]] = y_shard
    recv = torch.empty(world * M, widest, dtype=y_shard.dtype, device=y_shard.device)
    dist.all_gather_into_tensor(recv, send, group=group)
    parts = recv.view(world, M, widest)
    return torch.cat([parts[r, :, : n1 - n0] for r, (n0, n1) in enumerate(shards)], dim=1)


class ShardedLinear:
    """Y = X W^T with W split by output columns across the ranks of `group`.

    `compute(x, w_shard) -> y_shard` does this rank's part (default: the
    library's skinny_gemm); `forward` then gathers the full Y unless
    `gather=False`."""

    def __init__(self, w: torch.Tensor, rank: int, world: int, align: int = 128,
                 compute: Optional[Callable[[torch.Tensor, torch.Tensor], torch.Tensor]] = None, group=None,
                 out_div: int = 1):
        """out_div = 2 for the fused SiLU*mul weight: a block of W rows
        [n0, n1) yields output columns [n0 / 2, n1 / 2) (align must then be a
        multiple of 16, so every block holds whole gate/up pairs)."""
        if out_div == 2 and align % 16:
            raise ValueError("the SiLU*mul weight needs align to be a multiple of 16")
        self.N = w.shape[0]
        self.shards = column_shards(self.N, world, align)
        self.out_shards = [(n0 // out_div, n1 // out_div) for n0, n1 in self.shards]
        self.n0, self.n1 = self.shards[rank]
        self.w = w[self.n0:self.n1].contiguous()
        self.world, self.group, self.out_div = world, group, out_div
        if compute is None:
            from . import skinny_gemm as compute
        self.compute = compute

    def forward(self, x: torch.Tensor, gather: bool = True) -> torch.Tensor:
        if self.w.shape[0] > 0:
            y = self.compute(x, self.w)
        else:
            y = torch.empty(x.shape[0], 0, dtype=x.dtype, device=x.device)
        if not gather or self.world == 1:
            return y
        return gather_columns(y, self.out_shards, self.group)


def max_over_ranks(value: float, device=None, group=None) -> float:
    """The largest of the ranks' values (e.g. each rank's timed milliseconds)."""
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
