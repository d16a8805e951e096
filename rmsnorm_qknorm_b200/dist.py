"""Host-side plumbing for running the path on several GPUs (one process per GPU).

QK-Norm rows are independent, so the path partitions over tokens with no
collective on the data path: each rank either normalises its own batch (weak
scaling) or one contiguous shard of a shared batch (strong scaling).  The only
collectives are the timing ones: a barrier before and after the timed region
and a max-over-ranks reduction of the elapsed device time.
"""
from __future__ import annotations

import torch


def rank_seed(seed: int, rank: int) -> int:
    """Seed of a rank's synthetic batch (rank 0 keeps the workload's seed)."""
    return seed + 1000003 * rank


def shard_rows(total: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous [start, stop) rows of rank `rank` out of `world`; sizes differ by at most 1."""
    if world < 1 or not (0 <= rank < world) or total < 0:
        raise ValueError(f"bad shard request total={total} rank={rank} world={world}")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, group=None, device: str | torch.device = "cpu") -> float:
    """The maximum of `value` over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if group is None and not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def sum_over_ranks(value: float, group=None, device: str | torch.device = "cpu") -> float:
    """The sum of `value` over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if group is None and not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return float(t.item())
