"""Data-parallel replicas: which sequences a rank owns, and max-over-ranks timing.

Decode sequences (and prefill queries, once a sequence's compressed cache
exists) are independent, so ranks share no data: rank r of a run with
``per_rank`` sequences per GPU owns global sequences [r*per_rank, (r+1)*per_rank).
The only collective is the timing reduction.
"""
from __future__ import annotations


def shard(rank: int, per_rank: int) -> slice:
    """Global sequence range owned by `rank`."""
    if rank < 0 or per_rank <= 0:
        raise ValueError("rank must be >= 0 and per_rank > 0")
    return slice(rank * per_rank, (rank + 1) * per_rank)


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of `value` over all ranks of the default process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
