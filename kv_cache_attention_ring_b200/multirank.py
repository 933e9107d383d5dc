"""Multi-process plumbing for running the path on several GPUs (one process per GPU).

The path has no exchange step: rings, streams and heads are independent.  A job either
runs one replica of the whole workload per rank (weak scaling, what the benchmark does)
or splits the heads of each ring across ranks.  torch.distributed is used only for
barriers and for taking the maximum of per-rank timings; it works with the NCCL backend
on GPUs and with gloo on CPUs.
"""
from __future__ import annotations

import os


def dist_env() -> tuple[int, int, int]:
    """(rank, world_size, local_rank) from the torchrun environment (defaults 0, 1, 0)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard(n_items: int, rank: int, world: int) -> range:
    """Contiguous share of n_items for `rank`: sizes differ by at most one, lower ranks
    take the larger shares, and the shares tile [0, n_items) exactly."""
    if world < 1 or not 0 <= rank < world or n_items < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(n_items, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank float over the process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
