"""Multi-process plumbing for the engine (one process per GPU).

The forward pass has no exchange step: independent clips and streams are
split across ranks and each rank runs its own engine ("replicas"); the only
collective is the max-over-ranks reduction of the timed region.  Works with
any torch.distributed backend (NCCL on GPUs, gloo in the CPU tests)."""
from __future__ import annotations


def shard(n_units: int, rank: int, world: int):
    """Contiguous block of unit indices [lo, hi) owned by `rank` (the first
    n_units % world ranks take one extra unit)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(n_units, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of `value` over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def throughput(units_per_rank: float, ms_per_rank: float, device=None) -> float:
    """Whole-job throughput: units processed by all ranks / max-over-ranks
    time (units per second)."""
    total = sum_over_ranks(units_per_rank, device)
    slowest = max_over_ranks(ms_per_rank, device)
    return total / (slowest / 1000.0)
