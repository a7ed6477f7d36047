"""Host-side plumbing for running the hot path on several GPUs of one node.

Every step of the path (statistics, refresh, append, attention) is per head, with
no exchange between heads, so a layer shards by head with no collective on the
data path: rank r owns a contiguous block of heads and runs the same kernels on
its own cache.  The alternative is a replica per rank (each rank a whole layer).
`torch.distributed` is used only for the barrier and for reducing timings and
counts across ranks (NCCL on GPUs, gloo on CPU in the tests).
"""
from __future__ import annotations

import torch


def head_range(rank: int, world: int, heads: int) -> tuple[int, int]:
    """Heads [h0, h1) owned by `rank` of `world`: contiguous blocks whose sizes
    differ by at most one (the first heads % world ranks take one more)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if heads < world:
        raise ValueError(f"{heads} heads cannot be split over {world} ranks")
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def _reduce(x: float, op, device) -> float:
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x: float, device="cpu") -> float:
    """The largest value over all ranks (the slowest rank's time)."""
    import torch.distributed as dist

    return _reduce(x, dist.ReduceOp.MAX if dist.is_available() else None, device)


def sum_over_ranks(x: float, device="cpu") -> float:
    import torch.distributed as dist

    return _reduce(x, dist.ReduceOp.SUM if dist.is_available() else None, device)


def throughput(units_per_rank: float, seconds_per_rank: float, device="cpu") -> float:
    """Whole-job rate: the units all ranks processed over the slowest rank's time."""
    total = sum_over_ranks(units_per_rank, device)
    return total / max_over_ranks(seconds_per_rank, device)
