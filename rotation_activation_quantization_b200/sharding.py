"""Token sharding across ranks (one process per GPU) and the max-over-ranks timing rule.

SignRot's online path is independent per token row, so N GPUs split the rows: rank r of W owns
its own contiguous block of rows and no data-path collective is needed. The only collective is
the measurement's: the step time of a multi-GPU run is the slowest rank's.
"""
from __future__ import annotations


def shard_range(rank: int, world: int, total: int) -> tuple[int, int]:
    """Contiguous rows [t0, t1) of `total` owned by `rank` (sizes differ by at most one)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} not in a world of {world}")
    base, extra = divmod(int(total), world)
    t0 = rank * base + min(rank, extra)
    return t0, t0 + base + (1 if rank < extra else 0)


def weak_shard(rank: int, tokens_per_rank: int) -> tuple[int, int]:
    """Weak scaling: every rank processes its own `tokens_per_rank` rows of a larger stream."""
    return rank * tokens_per_rank, (rank + 1) * tokens_per_rank


def max_over_ranks(value: float, device=None) -> float:
    """All-reduce(MAX) of a scalar across the default process group (identity without one)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_all_ranks: int, max_seconds: float) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return units_all_ranks / max_seconds if max_seconds > 0 else float("inf")
