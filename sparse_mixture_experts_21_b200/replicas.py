"""Host-side plumbing for running the layer as data-parallel replicas.

Each rank routes and computes its own tokens against replicated experts; the
only exchange is the per-expert selection counts, summed over ranks before the
aux-loss-free bias update so every replica applies the same update and the
selection bias stays identical everywhere (the landscape page's point that the
balancing statistics should be global, not per micro-batch).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def all_reduce_counts(counts: torch.Tensor, out: torch.Tensor, group=None) -> torch.Tensor:
    """out = sum over ranks of counts (int32 [N]); counts is left untouched."""
    out.copy_(counts)
    dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out


def max_over_ranks(value: float, device, group=None) -> float:
    """The largest of each rank's value (used for step times)."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
