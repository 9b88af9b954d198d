"""Host-side helpers for running the path on several GPUs, one process per GPU.

The attention units are independent (a sequence's decode, a (batch, head) pair's
prefill), so ranks split the batch and never exchange data on the path; the only
collective is the timing reduction below.  Works with the gloo (CPU) and nccl
(GPU) backends of torch.distributed.
"""
from __future__ import annotations


def shard_range(n: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous [lo, hi) share of n units for `rank`; sizes differ by at most one."""
    if world <= 0 or not 0 <= rank < world or n < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def packed_shard(seqlens, rank: int, world: int) -> tuple[int, int, int, int]:
    """This rank's share of a decode batch whose caches are packed.

    Returns (lo, hi, row_lo, row_hi): sequences [lo, hi) of the batch
    (shard_range), whose cached tokens are rows [row_lo, row_hi) of the packed
    caches -- sequence b starts at the sum of the earlier non-negative lengths.
    The shard is itself a packed batch: q[lo:hi], caches[row_lo:row_hi],
    seqlens[lo:hi]."""
    lens = [max(int(x), 0) for x in seqlens]
    lo, hi = shard_range(len(lens), rank, world)
    row_lo = sum(lens[:lo])
    return lo, hi, row_lo, row_lo + sum(lens[lo:hi])


def max_over_ranks(x: float, device=None) -> float:
    """The maximum of x over all ranks (x itself without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def job_throughput(units_this_rank: float, ms_this_rank: float, device=None) -> float:
    """Whole-job throughput: all ranks' units divided by the slowest rank's time (units per second)."""
    total = sum_over_ranks(units_this_rank, device)
    slowest = max_over_ranks(ms_this_rank, device)
    return total / (slowest / 1e3)
