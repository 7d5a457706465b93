"""Expert-parallel MoE layer: each of W ranks holds N / W experts.

Orchestration only; every data-path step runs in the library's kernels:

  1. route and permute the rank's own tokens over all N experts (rows ordered by
     expert, hence by destination rank: they are the dispatch send buffer);
  2. exchange the expert offsets (all-gather) -- the counts travel before the rows;
  3. moe_ep_plan: split sizes, local expert offsets, regroup map (on the device);
     the split sizes are copied to the host for the all-to-all (the one
     synchronisation of the exchange);
  4. all-to-all of the rows; moe_rows_move regroups them by local expert;
  5. grouped SwiGLU FFN over the local experts;
  6. moe_rows_move back to arrival order; all-to-all back to the owning ranks;
  7. shared experts, combine; router statistics of the whole batch (every rank's
     sufficient statistics summed over ranks) and the bias update on the counts
     summed over ranks, so every rank keeps the same selection bias.

The exchange is an object with all_gather(t) -> [W, *t.shape],
all_to_all(out, inp, out_splits, in_splits) and all_reduce_sum(t); TorchDistExchange
runs them with torch.distributed (NCCL over NVLink on GPUs).  The phases are
separate methods so a caller can drive several ranks' layers in lock step.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _lib as L
from .layer import MoELayer
from .synth import Workload


class TorchDistExchange:
    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        out = torch.empty(self.world * t.numel(), dtype=t.dtype, device=t.device)
        self.dist.all_gather_into_tensor(out, t.contiguous().reshape(-1), group=self.group)
        return out.view((self.world,) + tuple(t.shape))

    def all_to_all(self, out, inp, out_splits, in_splits):
        self.dist.all_to_all_single(out, inp, output_split_sizes=list(out_splits),
                                    input_split_sizes=list(in_splits), group=self.group)

    def all_reduce_sum(self, t: torch.Tensor) -> torch.Tensor:
        self.dist.all_reduce(t, group=self.group)
        return t


class EPMoELayer:
    """Rank `rank` of `world`: routes its own T tokens over all N experts and computes
    the experts rank * N / W .. (rank + 1) * N / W - 1 for every rank's tokens."""

    def __init__(self, w: Workload, weights: dict, rank: int, world: int, device="cuda",
                 exchange=None, update_bias: bool = True, recv_factor: Optional[float] = None):
        if w.N % world != 0:
            raise ValueError(f"{w.N} experts do not divide over {world} ranks")
        if w.fp8 or w.mxfp8 or w.expert_choice or w.dtype != "bf16":
            raise ValueError("the expert-parallel layer runs bf16 token-choice routing")
        self.w, self.rank, self.world = w, rank, world
        self.El = w.N // world
        self.exchange = exchange
        dev = torch.device(device)
        lo, hi = rank * self.El, (rank + 1) * self.El
        # the single-rank layer supplies routing, permutation, shared experts, combine, stats;
        # it keeps only this rank's experts
        local = {k: v for k, v in weights.items() if k not in ("w1", "w3", "w2")}
        self.base = MoELayer(w, local, dev, update_bias=False)
        self.w1, self.w3, self.w2 = (weights[n][lo:hi].contiguous() for n in ("w1", "w3", "w2"))
        self.update_bias = update_bias and weights.get("bias") is not None
        # received rows: at most every rank's T * k rows (dropless, all to this rank's experts)
        cap = world * w.T * w.k if recv_factor is None else int(recv_factor * w.T * w.k)
        self.recv_cap = max(cap, 1)
        z = lambda *s, dtype=torch.bfloat16: torch.empty(s, dtype=dtype, device=dev)  # noqa: E731
        self.recv_x = z(self.recv_cap, w.d)
        self.x_loc = z(self.recv_cap, w.d)
        self.h_loc = z(self.recv_cap, w.f)
        self.y_loc = z(self.recv_cap, w.d)
        self.recv_y = z(self.recv_cap, w.d)
        self.send_splits = z(world, dtype=torch.int32)
        self.recv_splits = z(world, dtype=torch.int32)
        self.local_offsets = z(self.El + 1, dtype=torch.int32)
        self.regroup_map = z(self.recv_cap, dtype=torch.int32)
        self.counts_global = z(w.N, dtype=torch.int32)

    # ---------------------------------------------------------------- phases
    def dispatch_prepare(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        """Route and permute this rank's tokens; returns the offsets to all-gather."""
        b, c = self.base, self.base.cfg
        W = b.weights
        L.moe_route(c, x, W["w_gate"], W.get("logit_offset"), W.get("bias"), b.topk_idx, b.topk_w, b.lse,
                    b.p_partial, b.margin, b.ws, stream, shared_w=b.shared_w)
        L.moe_permute(c, x, b.topk_idx, b.counts, b.offsets, b.row_of_slot, b.token_of_row, b.x_perm,
                      b.n_dropped, b.ws, stream)
        return b.offsets

    def plan(self, offsets_all: torch.Tensor, stream=None):
        """Split sizes (host lists: send, receive) from every rank's offsets."""
        L.moe_ep_plan(offsets_all, self.world, self.rank, self.send_splits, self.recv_splits,
                      self.local_offsets, self.regroup_map, stream)
        send, recv = self.send_splits.cpu().tolist(), self.recv_splits.cpu().tolist()
        if sum(recv) > self.recv_cap:
            raise RuntimeError(f"{sum(recv)} rows received, capacity {self.recv_cap}")
        return send, recv

    def send_rows(self) -> torch.Tensor:
        return self.base.x_perm

    def local_compute(self, stream=None):
        """Regroup the received rows by local expert, run the local experts' grouped
        FFN, and put the results back in arrival order (self.recv_y)."""
        w = self.w
        n = self.local_offsets[self.El:]                      # device scalar: rows received
        L.moe_rows_move(self.recv_x, self.regroup_map, n, self.x_loc, scatter=True, stream=stream)
        L.moe_grouped_ffn(self.base.cfg, self.x_loc, self.recv_cap, self.local_offsets, self.El,
                          self.w1, self.w3, self.w2, w.f, self.h_loc, self.y_loc, stream)
        L.moe_rows_move(self.y_loc, self.regroup_map, n, self.recv_y, scatter=False, stream=stream)

    def stats_partial(self, stream=None) -> torch.Tensor:
        """This rank's sufficient statistics (fp64 [3N + 5]), to be summed over ranks."""
        b = self.base
        L.moe_router_stats_partial(b.cfg, b.counts, b.offsets, b.p_partial, b.lse, b.n_dropped, b.stats_part,
                                   margin=b.margin, stream=stream)
        return b.stats_part

    def finish(self, x: torch.Tensor, stream=None, partial_sum: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Shared experts, combine (base.y_perm holds the returned rows), statistics
        and bias update.  With partial_sum (the sum over ranks of stats_partial())
        the statistics are the whole batch's and the bias update uses the summed
        counts; without it, this rank's statistics and no bias update."""
        b, c, w = self.base, self.base.cfg, self.w
        W = b.weights
        shared = None
        if b.fs > 0:
            L.moe_grouped_ffn(c, x, w.T, b.shared_offsets, 1, W["ws1"], W["ws3"], W["ws2"], b.fs, b.hs, b.ys,
                              stream)
            shared = b.ys
        L.moe_combine(c, b.y_perm, b.row_of_slot, b.topk_w, shared, b.y, stream, shared_w=b.shared_w)
        if partial_sum is None:
            L.moe_router_stats(c, b.counts, b.offsets, b.p_partial, b.lse, b.n_dropped, W.get("bias"), w.alpha,
                               w.z_coef, b.stats, b.f_out, b.p_out, stream, margin=b.margin)
        else:
            L.moe_router_stats_finalize(c, partial_sum, W.get("bias"), w.alpha, w.z_coef, b.stats, b.f_out,
                                        b.p_out, self.counts_global, stream)
            if self.update_bias:
                L.moe_bias_update(c, self.counts_global, W["bias"], w.bias_rate, 0.0, stream)
        return b.y

    # ---------------------------------------------------------------- one rank, real exchange
    def forward(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        ex = self.exchange
        offsets_all = ex.all_gather(self.dispatch_prepare(x, stream))
        send, recv = self.plan(offsets_all, stream)
        ex.all_to_all(self.recv_x[:sum(recv)], self.base.x_perm[:sum(send)], recv, send)
        self.local_compute(stream)
        ex.all_to_all(self.base.y_perm[:sum(send)], self.recv_y[:sum(recv)], send, recv)
        part = ex.all_reduce_sum(self.stats_partial(stream))
        return self.finish(x, stream, part)

    def kernel_launches(self) -> int:
        # route (+ split), permute (4), plan, two row moves, local FFN (2), combine, stats (2), bias
        n = 1 + 1 + 4 + 1 + 2 + 2 + 1 + 2
        n += 2 if self.base.fs > 0 else 0
        return n + (1 if self.update_bias else 0)
