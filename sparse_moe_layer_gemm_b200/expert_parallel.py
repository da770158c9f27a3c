"""Expert parallelism for the MoE layer: each rank holds a contiguous shard of
the routed experts (rank 0 also holds the shared expert), routes every token
over all experts, computes the pairs that selected its own experts, and an
all-reduce over the ranks sums the partial outputs into the layer's output
(the same T tokens on every rank).

The split and the reduction are host logic; every arithmetic step of a
shard's forward runs in libmoe.so (``moe_create_shard``).  The collective is
``torch.distributed.all_reduce`` over the process group: NCCL over NVLink
between GPUs, gloo between CPU processes in the tests.
"""
from __future__ import annotations

from typing import Dict, Optional, Tuple

import torch
import torch.distributed as dist


def shard_range(num_experts: int, world: int, rank: int) -> Tuple[int, int]:
    """(first, count) of rank's routed experts: contiguous, sizes differing by
    at most one, together covering [0, num_experts) once."""
    if world < 1 or not 0 <= rank < world or num_experts < world:
        raise ValueError(f"cannot split {num_experts} experts over {world} ranks (rank {rank})")
    first = rank * num_experts // world
    return first, (rank + 1) * num_experts // world - first


def holds_shared(rank: int) -> bool:
    """The shared expert is computed once, on rank 0."""
    return rank == 0


def reduce_partials(out: torch.Tensor, group=None) -> torch.Tensor:
    """Sums the ranks' partial outputs in place (no-op without a process
    group of more than one rank)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out


class ExpertParallelMoE:
    """The layer split over the ranks of `group` (default: the world)."""

    def __init__(self, cfg, group=None):
        from .binding import MoeLayer
        self.group = group
        inited = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if inited else 1
        self.rank = dist.get_rank(group) if inited else 0
        first, count = shard_range(cfg.num_experts, self.world, self.rank)
        self.shard = (first, count, holds_shared(self.rank))
        self.layer = MoeLayer(cfg, self.shard)

    def load_inputs(self, inp: Dict[str, torch.Tensor]):
        """The full [E, ...] expert tensors on every rank; the library packs
        only this rank's slice."""
        self.layer.load_inputs(inp)

    def load_shard_inputs(self, inp: Dict[str, torch.Tensor]):
        """This rank's experts only ([count, ...], e.g. from
        workloads.make_shard_inputs): a rank holds 1/N of the expert bytes."""
        self.layer.load_shard_weights(inp["router_w"], inp["router_bias"], inp["w_gate"],
                                      inp["w_up"], inp["w_down"], inp.get("sh_gate"),
                                      inp.get("sh_up"), inp.get("sh_down"))

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        return reduce_partials(self.layer.forward(x, out), self.group)

    def close(self):
        self.layer.close()
