"""Host-side helpers of the multi-GPU (data-parallel) path.

The HiF4 path partitions without any exchange: quantization units are
independent, and the linear layer shards over tokens with the weights
replicated.  One process per GPU; torch.distributed is used only for the
start/stop barrier and for taking the slowest rank's time.
"""
from __future__ import annotations


def token_shard(total: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous, balanced [start, stop) token range of `rank` (strong scaling)."""
    if world < 1 or not 0 <= rank < world or total < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def rank_seed(base: int, rank: int) -> int:
    """Seed of a rank's own batch (weak scaling: every rank draws its own tokens)."""
    return base + 1009 * rank


def max_over_ranks(value: float, device=None) -> float:
    """Largest `value` over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None) -> None:
    """All ranks meet, then this rank's device work is drained."""
    import torch
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()
    if device is not None and torch.cuda.is_available():
        torch.cuda.synchronize(device)


def aggregate_throughput(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return units_per_rank * world / max_seconds
