"""Data-parallel probe step: one exchange of two numbers per step.

The path shards over prompts.  Every replica holds the full frozen weights and
the same bank, and draws identical U/V from the counter stream, so nothing
but the objective needs to cross GPUs.  Each replica scores its own prompts
(both candidates), sums its paired differences, and one all-reduce of
{sum_i (L+_i - L-_i), n_prompts} gives every replica the same
c = sum / n / (2 eps); the bank update that follows is identical everywhere.
This is the estimator of "Zeroth-Order Fine-Tuning Was an Inference Workload
All Along" (section "Why ZO Fine-Tuning Is Really Scoring") over the union of
the replicas' prompts.
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

from . import workload as wl


def shard_batch(batch: wl.Batch, rank: int, world: int) -> wl.Batch:
    """Contiguous shard of the prompts (and foreground rows) for one replica."""
    def cut(n):
        per, extra = divmod(n, world)
        lo = rank * per + min(rank, extra)
        return lo, lo + per + (1 if rank < extra else 0)
    a, b = cut(len(batch.prompts))
    fa, fb = cut(len(batch.fg_prompts))
    return wl.Batch(batch.prompts[a:b], batch.target_lens[a:b], batch.fg_prompts[fa:fb],
                    batch.fg_target_lens[fa:fb])


def allreduce_sums(sums: torch.Tensor, group: Optional[dist.ProcessGroup] = None) -> torch.Tensor:
    """In-place SUM of the per-replica {sum of paired differences, prompt count} (float64 [2])."""
    if sums.dtype != torch.float64 or sums.numel() != 2:
        raise ValueError("sums must be a float64 tensor of two elements")
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(sums, op=dist.ReduceOp.SUM, group=group)
    return sums


def dp_step(handle, lr: float, sums: torch.Tensor, group: Optional[dist.ProcessGroup] = None,
            want_c: bool = False):
    """zo_objective_sums on this replica, one all-reduce, then zo_step_from_sums."""
    handle.zo_objective_sums(sums)
    allreduce_sums(sums, group)
    return handle.zo_step_from_sums(lr, sums, want_c=want_c)
