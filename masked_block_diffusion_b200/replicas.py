"""Host plumbing for running independent requests as replicas across ranks.

Requests of a batch are independent (no exchange between them in the denoising pass),
so several GPUs serve them as replicas: each rank holds the full model and a disjoint
share of the requests. The only collectives are timing ones: a barrier around the timed
region and the maximum of the ranks' times.
"""

from __future__ import annotations

from typing import List


def shard_requests(n_requests: int, world: int, rank: int) -> List[int]:
    """The request ids rank `rank` serves: round-robin, disjoint, covering all."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world / rank")
    return list(range(rank, n_requests, world))


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of `value` over the ranks of the default process group (identity when
    torch.distributed is not initialised). device: where the reduction tensor lives
    ("cuda" for NCCL, "cpu" for gloo)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: int, world: int, max_seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    if max_seconds <= 0:
        raise ValueError("time must be positive")
    return units_per_rank * world / max_seconds
