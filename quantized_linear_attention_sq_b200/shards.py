"""Data-parallel plumbing for several GPUs (one process per GPU).

The decode step of one request touches only that request's state, so a
multi-GPU job shards requests across ranks with no collective on the data
path: every rank owns a full batch of its own requests (weak scaling). The
only collectives are the ones the measurement needs: a barrier around the
timed region and the maximum of the ranks' device times.
"""
from __future__ import annotations


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of the synthetic workload shard owned by `rank` (distinct
    requests on every rank)."""
    return base_seed + rank


def max_over_ranks(x: float, dist=None, device=None) -> float:
    """Maximum of a per-rank scalar over all ranks (the slowest rank sets a
    multi-GPU time). `dist` is torch.distributed with an initialised process
    group, or None for a single process."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: int, steps: int, max_ms: float, world: int) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time (units per second)."""
    return world * units_per_rank * steps / (max_ms / 1e3)
