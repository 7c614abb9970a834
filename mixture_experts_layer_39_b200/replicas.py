"""Host plumbing for running the layer as replicas, one process per GPU.

Every rank runs the whole layer on its own tokens with all experts resident,
so the layer itself never exchanges rows between GPUs.  What a
data-parallel job still needs across ranks is small and lives here:

  world()          rank layout from the launcher's environment
                   (WORLD_SIZE, RANK, LOCAL_RANK);
  max_over_ranks() the slowest rank's value of a device-timed duration;
  sum_load_stats() the router's load statistics [counts | probability sums]
                   (2E fp32) added over ranks, so that the load-balancing
                   loss is formed over the global batch (the v2 router's
                   global load balancing: Olmo-core 3 introduction page,
                   section 4).  It moves 2E floats per step.

All three work with any torch.distributed backend (NCCL on GPUs, gloo on
the host) and are no-ops without an initialised process group.
"""
from __future__ import annotations

import os
from typing import Callable

import torch
import torch.distributed as dist


def world() -> tuple[int, int, int]:
    """(world size, rank, local rank) from the launcher's environment."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _active() -> bool:
    return dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1


def max_over_ranks(value: float, device: torch.device | str = "cpu") -> float:
    """The largest `value` over all ranks (every rank must call it)."""
    if not _active():
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_load_stats(stats: torch.Tensor) -> torch.Tensor:
    """Adds the load statistics of all ranks into `stats`, in place, and
    returns it (every rank must call it)."""
    if _active():
        dist.all_reduce(stats, op=dist.ReduceOp.SUM)
    return stats


def global_stats_reducer(tokens_per_rank: int) -> Callable[[torch.Tensor], int]:
    """For MoELayer(aux_reduce=...): sums the statistics over ranks and
    returns the global batch's token count (every rank the same T)."""
    def reduce(stats: torch.Tensor) -> int:
        sum_load_stats(stats)
        ws = dist.get_world_size() if _active() else 1
        return tokens_per_rank * ws
    return reduce
