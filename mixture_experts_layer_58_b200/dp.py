"""Data-parallel exchanges of the DeepSeekMoE layer.

Forward: each rank routes its own batch; the auxiliary-loss-free bias update
(DeepSeek-V3 technical report summary, Method §2: b_i -= gamma when expert i is
overloaded, += gamma when underloaded, at the end of a step) needs the load of
the whole step, so the per-expert counts are summed over ranks before every
rank applies the same update to its replica of the bias. That is the only
exchange of an inference step.

Training: the replicated weights need the gradient of the global loss, so the
weight and centroid gradients are averaged over ranks after the backward.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def sync_load(counts: torch.Tensor, tokens_per_rank: int, group=None) -> int:
    """Sum `counts` ([N_r] int32, any device the backend supports) over the
    ranks of `group` in place and return the global token count. Every rank
    must hold the same number of tokens (the benchmark's weak-scaling batch)."""
    dist.all_reduce(counts, op=dist.ReduceOp.SUM, group=group)
    return int(tokens_per_rank) * dist.get_world_size(group)


def allreduce_grads(grads, group=None, average: bool = True) -> None:
    """Data-parallel training: sum each gradient tensor in `grads` over the
    ranks of `group` in place (NCCL on the GPU, any backend for host tensors),
    then divide by the number of ranks when `average` (each rank's loss a mean
    over its own tokens, the global loss the mean over ranks). Every rank must
    pass the same tensors in the same order."""
    world = dist.get_world_size(group)
    for g in grads:
        if g is None:
            continue
        dist.all_reduce(g, op=dist.ReduceOp.SUM, group=group)
        if average and world > 1:
            g.div_(world)
