"""Multi-GPU plumbing for the relation-KL path.

Every (relation, batch, head) unit is independent: Phase 1, Phase 2 and the
gradients of a head need only that head's projections (LinearARD notes,
关键设计 1 and 3: the maps, statistics and gradients are per head).  Two ways
to use several GPUs follow from that:

* weak scaling: each rank runs its own batch of units (``rank_workload``);
  nothing crosses ranks on the data path;
* one job split across ranks (``partition_units`` / ``rank_slices``): the
  units of ONE workload are cut into contiguous, equal-work slices, one per
  rank; each rank runs its slice in one grouped launch per phase and keeps
  its heads' gradients; the job's loss is the sum of the ranks' losses, one
  scalar all-reduce (``all_reduce_loss``).

The only other cross-rank step is the timing reduction of a benchmark (the
job's time is the slowest rank's).
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


def partition_units(units, world: int, rank: int):
    """The slice of one job's units that ``rank`` of ``world`` runs.

    ``units`` lists (relation, count) in launch order, count = B * H of that
    relation; a relation's units are its flattened (b, h) indices, which are
    contiguous in a [B, H, n, d] tensor.  Units of one grouped call share n, so
    every unit costs the same (n(n+1)/2 causal logits): an equal-work split is
    an equal-count split.  The job's U units, relation after relation, are cut
    at floor(r * U / world); rank r takes [floor(r U / G), floor((r+1) U / G)),
    so the slices are contiguous, disjoint, cover every unit once, and differ
    in size by at most one unit.  Returns [(relation, lo, hi)] with the
    half-open range of flattened (b, h) indices per relation the slice touches
    (empty if the rank gets no unit)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    total = sum(c for _, c in units)
    start, stop = rank * total // world, (rank + 1) * total // world
    out, base = [], 0
    for rel, count in units:
        lo, hi = max(start, base), min(stop, base + count)
        if lo < hi:
            out.append((rel, lo - base, hi - base))
        base += count
    return out


def rank_slices(w, world: int, rank: int):
    """``partition_units`` for a workload: its relations in order, B * H units each."""
    return partition_units([(r, w.B * w.heads[r]) for r in w.relations], world, rank)


def slice_heads(t, lo: int, hi: int):
    """Units [lo, hi) of a [B, H, ...] tensor as a contiguous [1, hi - lo, ...] view
    (the flattened (b, h) index is contiguous in memory)."""
    flat = t.reshape(t.shape[0] * t.shape[1], *t.shape[2:])
    return flat[lo:hi].unsqueeze(0)


def all_reduce_loss(loss):
    """Sum a rank's loss tensor (1 element, on its device) over all ranks, in
    place: the job's loss when each rank ran its own slice of the units.  A
    no-op for one rank."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(loss, op=dist.ReduceOp.SUM)
    return loss


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


def job_rate(units_per_step: int, steps: int, max_elapsed_ms: float) -> float:
    """Whole-job throughput when the ranks split one job: its units / the slowest rank's time."""
    return units_per_step * steps / (max_elapsed_ms / 1e3)
