"""Multi-GPU plumbing for data-parallel use of the relation-KL path.

Every (relation, batch, head) unit is independent, so a multi-GPU job gives
each rank its own batch of units and needs no collective on the data path.
The only cross-rank steps are the timing reduction of a benchmark (max over
ranks) and, for a training loop, the sum of the scalar losses.
"""
from __future__ import annotations

import dataclasses
import os
from datetime import timedelta


def env_ranks():
    """(rank, world size, local rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, device=None, timeout_s: int = 120):
    """Initialise the default process group from the environment (no-op for one rank)."""
    import torch.distributed as dist
    _, world, _ = env_ranks()
    if world > 1 and not dist.is_initialized():
        kw = {"timeout": timedelta(seconds=timeout_s)}
        if device is not None:
            kw["device_id"] = device
        dist.init_process_group(backend, **kw)
    return world


def rank_workload(w, rank: int):
    """The workload a rank runs: same shapes, its own seed (its own batch)."""
    return dataclasses.replace(w, seed=w.seed + 1000 * rank)


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a scalar over all ranks (a rank's time -> the job's time)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    """Sum of a scalar over all ranks (e.g. the job's total loss)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def aggregate_rate(units_per_step_per_rank: int, steps: int, world: int, max_elapsed_ms: float) -> float:
    """Whole-job throughput under weak scaling: all ranks' units / the slowest rank's time."""
    return units_per_step_per_rank * steps * world / (max_elapsed_ms / 1e3)
