"""Data-parallel exchange of the DeepSeekMoE layer: the only cross-rank step.

Each rank routes its own batch; the auxiliary-loss-free bias update (DeepSeek-V3
technical report summary, Method §2: b_i -= gamma when expert i is overloaded,
+= gamma when underloaded, at the end of a step) needs the load of the whole
step, so the per-expert counts are summed over ranks before every rank applies
the same update to its replica of the bias.
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
