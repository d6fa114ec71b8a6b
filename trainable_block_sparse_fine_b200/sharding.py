"""Multi-GPU sharding of the VSA2 hot path.

The router, the per-sequence TopK (its budget belongs to one (batch, head)) and the block-sparse
attention are independent per (batch, head), so ranks split the (b, h) units and never exchange
data on the path. Only the host-side timing takes a maximum over ranks.
"""
from __future__ import annotations


def shard_units(batch: int, heads: int, rank: int, world: int) -> list[tuple[int, int]]:
    """(b, h) pairs owned by `rank`: a contiguous, balanced split of the batch*heads units
    (the first batch*heads % world ranks take one extra unit)."""
    if world < 1 or not (0 <= rank < world):
        raise ValueError("need 0 <= rank < world")
    total = batch * heads
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    count = base + (1 if rank < extra else 0)
    return [divmod(u, heads) for u in range(start, start + count)]


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank scalar over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
