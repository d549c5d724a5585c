"""Host-side plumbing for running the forward on several GPUs of one node.

Every (b, h) attention problem is independent, so a multi-GPU run is a set
of replicas: rank r owns its own batch shard (the workload's B heads drawn
from a rank-specific seed), there is no collective on the data path, and
only the timing is combined (max over ranks).
"""
from __future__ import annotations

import dataclasses

import torch

from .synth import Workload


def shard_workload(w: Workload, world: int, rank: int) -> Workload:
    """Rank ``rank``'s shard under weak scaling: same per-GPU shape, its own
    seed, so the global batch is ``world * w.B`` distinct problems."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    if world == 1:
        return w
    return dataclasses.replace(w, seed=w.seed + 100003 * rank,
                               name=f"{w.name} [shard {rank}/{world}]")


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank scalar (e.g. elapsed ms) over the process group."""
    if world == 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
