"""Host-side plumbing for running the decoders on several GPUs.

Decoding shards with no exchange step: every LZ4 block, zero-run chunk,
row, matrix and layer decodes independently. Ranks therefore take disjoint
contiguous ranges of units and never exchange data; the only collectives
are the timing reductions (one scalar each, outside the data path).
"""
from __future__ import annotations


def shard_range(n_units: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous, balanced share [start, end) of ``n_units`` for ``rank``
    (the first ``n_units % world`` ranks take one extra unit)."""
    if world < 1 or not 0 <= rank < world or n_units < 0:
        raise ValueError("need 0 <= rank < world and n_units >= 0")
    base, extra = divmod(n_units, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def shard_blocks(block_offsets, rank: int, world: int):
    """This rank's share of an LZ4 stream given by its n_blocks + 1 byte
    offsets: (first block, block count, byte offsets rebased to the share,
    first compressed byte)."""
    n_blocks = len(block_offsets) - 1
    b0, b1 = shard_range(n_blocks, rank, world)
    base = int(block_offsets[b0])
    rebased = [int(o) - base for o in block_offsets[b0:b1 + 1]]
    return b0, b1 - b0, rebased, base


def reduce_max(value: float, group=None, device=None) -> float:
    """Max of a scalar over the ranks of ``group`` (identity without a
    process group): the job's time is its slowest rank's."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def reduce_sum(value: float, group=None, device=None) -> float:
    """Sum of a scalar over the ranks (the whole job's decoded bytes)."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return float(t.item())
