"""Token sharding across ranks (one process per GPU), the calibration merge and the
max-over-ranks timing rule.

SignRot's online path is independent per token row, so N GPUs split the rows: rank r of W owns
its own contiguous block of rows and no data-path collective is needed. Calibration (the
abstract's "single calibration forward pass") over a calibration set split across ranks has one
real exchange: every rank folds its own rows into the per-channel keys (max |x|, first token,
sign), then one all-reduce(MAX) of the n keys gives every rank the keys of the whole set, from
which each rank takes the same argmax and builds the same sign vector. The other collective is
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


def merge_calibration(ws, group=None):
    """All-reduce(MAX), in place, of the per-channel calibration keys ws [n] (int64 storage).

    A key is |x| as fp32 bits << 32 | (2^31 - 1 - t) << 1 | sign, with t the token's index in the
    whole calibration set, so the maximum over ranks is the key the whole set would have given:
    the largest magnitude, its first token on a tie, and that value's sign. |x| of a finite
    value is below 2^31, so every key is a non-negative int64 and the signed maximum is the
    unsigned one. Identity without a process group (or with one rank).
    """
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return ws
    dist.all_reduce(ws, op=dist.ReduceOp.MAX, group=group)
    return ws
