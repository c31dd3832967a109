"""Multi-GPU plumbing for the PD-SSM scan: one process per GPU.

The recurrence is independent per (batch, head) sequence, so the natural
split is data parallel: each rank owns a contiguous block of batch rows and
runs the whole path on them with no data-path collective.  The only
cross-rank operations are the timing barrier and the max-over-ranks of the
measured time (torch.distributed, NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations


def batch_shard(B: int, world: int, rank: int) -> tuple[int, int]:
    """[start, stop) of the batch rows owned by `rank`; blocks differ in size
    by at most one row and cover 0..B-1 exactly once."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(B, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar (e.g. a measured time) over all ranks."""
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
