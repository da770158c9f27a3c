"""Host logic of the multi-GPU run: one replica of the layer per rank, each on
its own batch (the layer is token-wise independent, so ranks exchange no data
on the path).  ``torch.distributed`` serves only the barrier and the
max-over-ranks timing reduction."""
from __future__ import annotations

from dataclasses import replace

import torch
import torch.distributed as dist

from .workloads import Workload


def rank_batch_workload(wl: Workload, rank: int) -> Workload:
    """The workload whose x a rank draws: same weights everywhere (seed of the
    weights unchanged), a different batch per rank."""
    return replace(wl, seed=wl.seed + rank)


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of `value` over all ranks (the value itself without a
    process group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: the tokens all ranks processed per step divided by
    the slowest rank's step time."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)
