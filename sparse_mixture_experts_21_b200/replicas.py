"""Host-side plumbing for running the layer as data-parallel replicas.

Each rank routes and computes its own tokens against replicated experts; the
only exchange is each rank's vector of router sufficient statistics (per-expert
counts, kept counts and affinity sums, sum of lse^2, tokens, drops, near-ties),
summed over ranks so the statistics and the aux-loss-free bias update are those
of the whole batch and every replica applies the same update (the landscape
page's point that the balancing statistics should be global, not per
micro-batch).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def all_reduce_counts(counts: torch.Tensor, out: torch.Tensor, group=None) -> torch.Tensor:
    """out = sum over ranks of counts (int32 [N]); counts is left untouched."""
    out.copy_(counts)
    dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out


def all_reduce_sum(t: torch.Tensor, group=None) -> torch.Tensor:
    """t <- sum over ranks of t, in place."""
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return t


def max_over_ranks(value: float, device, group=None) -> float:
    """The largest of each rank's value (used for step times)."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
