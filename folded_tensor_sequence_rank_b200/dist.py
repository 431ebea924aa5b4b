"""Host-side plumbing for running TSP ranks one per GPU.

Each process (one per GPU, launched by torchrun) runs TSP rank
``global_rank % D`` of the layer as an independent problem; the only
collectives are the barrier around timed regions and the max over ranks of a
measured time, so a job's time is that of its slowest rank.
"""
from __future__ import annotations

import os


def world_info():
    """(world_size, global_rank, local_rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def tsp_rank_for(global_rank: int, D: int) -> int:
    """The TSP rank a process runs: processes cycle through the D ranks."""
    if D < 1:
        raise ValueError("D must be positive")
    return global_rank % D


def max_over_ranks(values, device=None):
    """Element-wise maximum of a list of floats over all processes (identity when
    torch.distributed is not initialised or has one rank)."""
    import torch
    import torch.distributed as dist
    vals = [float(v) for v in values]
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()
