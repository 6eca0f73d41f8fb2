"""Output-row (N) sharding of a packed linear over the ranks of a process group.

No page describes tensor parallelism; the partition is this library's own.
Rank r of ``world`` owns the weight rows ``r * Nl .. r * Nl + Nl - 1``, where
``Nl`` is ``ceil(N / world)`` rounded up to a multiple of 16 (the decode
kernel's row tile); rows past N are zero codes with scale 1 and give zero
outputs.  Each rank keeps only its rows (packed) and their scales, so a
matrix's bytes are split ``world`` ways.

A call with the replicated input x runs the rank's linear on the library's
kernels (``y_r = x @ W_r^T``, [M, Nl]), then one all-gather over the process
group (NCCL on GPUs) collects the ``y_r`` rank after rank as blocks
[world, M, Nl]; for M = 1 these already are y, for M > 1 ``mpw_gather_shards``
interleaves them into y [M, N].  Every rank takes the same collective in the
same order.  No memory of another GPU is read by a kernel here: the only
transfer is the library collective.
"""
from __future__ import annotations

from dataclasses import dataclass

ROW_TILE = 16


def rows_per_rank(N: int, world: int, align: int = ROW_TILE) -> int:
    """Nl: ceil(N / world) rounded up to a multiple of ``align``."""
    if N < 1 or world < 1 or align < 1:
        raise ValueError("N, world and align must be positive")
    per = -(-int(N) // int(world))
    return -(-per // align) * align


def rank_rows(N: int, world: int, rank: int, align: int = ROW_TILE):
    """(n0, n1): the rows of W that rank owns (n1 <= N; empty when n0 >= N)."""
    if not 0 <= rank < world:
        raise ValueError("rank outside the group")
    Nl = rows_per_rank(N, world, align)
    n0 = min(rank * Nl, N)
    return n0, min(n0 + Nl, N)


def shard_packed(packed, scales, N: int, world: int, rank: int, align: int = ROW_TILE):
    """Rank's rows of a packed matrix: (packed_r [Nl, row_bytes] with zero
    rows past N, scales_r [Nl] with 1.0 there).  Works on tensors of any
    device; the copies stay on it."""
    import torch

    Nl = rows_per_rank(N, world, align)
    n0, n1 = rank_rows(N, world, rank, align)
    pr = torch.zeros((Nl, packed.shape[1]), dtype=packed.dtype, device=packed.device)
    sr = torch.ones((Nl,), dtype=scales.dtype, device=scales.device)
    if n1 > n0:
        pr[: n1 - n0].copy_(packed[n0:n1])
        sr[: n1 - n0].copy_(scales[n0:n1])
    return pr, sr


@dataclass
class ShardedLinear:
    """One rank's share of a packed linear (see the module docstring)."""

    packed: object     # uint8 [Nl, row_bytes]
    scales: object     # fp32 [Nl]
    N: int
    K: int
    bits: int
    world: int
    rank: int
    layout: str = "canonical"

    @property
    def Nl(self) -> int:
        return self.packed.shape[0]

    @classmethod
    def from_full(cls, packed, scales, N: int, K: int, bits: int, world: int, rank: int,
                  layout: str = "canonical", align: int = ROW_TILE):
        pr, sr = shard_packed(packed, scales, N, world, rank, align)
        return cls(pr, sr, int(N), int(K), int(bits), int(world), int(rank), layout)


def _local_qlinear(x, lin: ShardedLinear):
    from . import qlinear

    return qlinear(x, lin.packed, lin.scales, lin.bits, layout=lin.layout)


def _gather_columns(blocks, world: int, M: int, Nl: int, N: int, y):
    from . import gather_shards

    return gather_shards(blocks, world, M, Nl, N, y=y)


def qlinear_sharded(x, lin: ShardedLinear, y=None, group=None, local=None, reorder=None):
    """y [M, N] = x @ W^T from every rank's share: the rank's own linear, one
    all-gather of the outputs over ``group``, then the column order.

    ``local(x, lin) -> y_r [M, Nl]`` and ``reorder(blocks, world, M, Nl, N,
    y)`` default to the library's kernels (qlinear, gather_shards); they are
    parameters so that the partition and the gather order can be exercised
    on CPU ranks."""
    import torch
    import torch.distributed as dist

    local = local or _local_qlinear
    reorder = reorder or _gather_columns
    M = x.shape[0]
    Nl, N, world = lin.Nl, lin.N, lin.world
    y_r = local(x, lin)
    if tuple(y_r.shape) != (M, Nl):
        raise ValueError("local output must be [M, Nl]")
    if world == 1:
        blocks = y_r.reshape(-1)
    else:
        blocks = torch.empty((world * M * Nl,), dtype=y_r.dtype, device=y_r.device)
        dist.all_gather_into_tensor(blocks, y_r.contiguous().reshape(-1), group=group)
    if M == 1:
        # the blocks already are y
        if y is None:
            return blocks[:N].view(1, N)
        y.view(-1).copy_(blocks[:N])
        return y
    if y is None:
        y = torch.empty((M, N), dtype=y_r.dtype, device=y_r.device)
    reorder(blocks, world, M, Nl, N, y)
    return y
