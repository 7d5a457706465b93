"""Expert-parallel MoE layer: each of W ranks holds N / W experts.

Orchestration only; every data-path step runs in the library's kernels:

  1. route and permute the rank's own tokens over all N experts (rows ordered by
     expert, hence by destination rank: they are the dispatch send buffer);
  2. exchange the expert offsets (all-gather) -- the counts travel before the rows;
  3. plan the exchange on the host (the one synchronisation of a forward): every
     rank derives the same plan from the all-gathered offsets.  The rows a rank
     receives are bounded by its receive buffer (recv_factor * T * k rows, at
     least T): a destination's (source, expert) pieces are packed, in expert then
     source order, into rounds that each fit the buffer, and every rank runs as
     many rounds as the busiest destination needs.  (With the peer exchange and
     device_plan=True the buffer holds every row a rank can receive, one round
     always suffices, and the offsets never leave the device.);
  4. per round: all-to-all of the round's rows; moe_ep_plan + moe_rows_move regroup
     them by local expert; grouped SwiGLU FFN over the local experts; moe_rows_move
     back to arrival order; all-to-all back into the owning ranks' y_perm;
  5. shared experts, combine; router statistics of the whole batch (every rank's
     sufficient statistics summed over ranks) and the bias update on the counts
     summed over ranks, so every rank keeps the same selection bias.

With a real exchange (forward) rounds use two buffer sets: round r + 1's dispatch
is issued before round r's expert compute and round r's return right after it, so
the transfers overlap the grouped GEMMs ([Practice] "通信优化按什么顺序做": overlap
the dispatch with expert compute).

With peer=True the rows travel over NVLink peer memory instead: every rank maps the
other ranks' receive buffers once, and per round moe_ep_peer_plan gives each of its
rows its address in the owning rank's receive buffer (local-expert order, so no
regroup pass), moe_ep_peer_dispatch stores x rows straight there (the permutation's
gather and the dispatch in one kernel: the expert-ordered copy of x is never
written), a barrier, the local grouped FFN in place on the receive buffer (the shared
expert fused into round 0's launches), a barrier, and the results are read back by
the owning ranks' kernels: moe_combine_peer loads them from the peers' buffers
directly when there is one round, moe_ep_peer_collect pulls each round's into y_perm
otherwise.  No kernel waits for another rank's; the barriers are collectives on the
compute stream.

The exchange is an object with all_gather(t) -> [W, *t.shape],
all_to_all(out_list, in_list, async_op) (lists of per-rank tensors; async_op returns
a handle with wait()) and all_reduce_sum(t); for peer=True also barrier() (stream
ordered), peer_addresses(t) -> [W] device addresses of every rank's t (collective;
t has the same shape everywhere) and release_peer(address).  TorchDistExchange runs
them with torch.distributed (NCCL over NVLink on GPUs) and the library's CUDA IPC
mapping.  The phases are separate methods so a caller can drive several ranks'
layers in lock step.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Optional

import numpy as np
import torch

from . import _lib as L
from .layer import MoELayer
from .synth import Workload


class _Works:
    """Handle of a batch of point-to-point operations."""

    def __init__(self, works):
        self.works = works

    def wait(self):
        for w in self.works:
            w.wait()


class TorchDistExchange:
    """device: where barrier() keeps its one-element flag (default: the current CUDA
    device; "cpu" for a gloo group on the host)."""

    def __init__(self, group=None, device=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.device = device

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        out = torch.empty(self.world * t.numel(), dtype=t.dtype, device=t.device)
        self.dist.all_gather_into_tensor(out, t.contiguous().reshape(-1), group=self.group)
        return out.view((self.world,) + tuple(t.shape))

    def all_to_all(self, out_list, in_list, async_op: bool = False):
        """out_list[s] <- what rank s sends here; in_list[d] -> rank d.  Batched
        point-to-point sends and receives (one grouped call under NCCL); a rank's own
        slice is a local copy and empty slices are skipped on both ends."""
        dist = self.dist
        ops = []
        for peer in range(self.world):
            gpeer = peer if self.group is None else dist.get_global_rank(self.group, peer)
            if peer == self.rank:
                if out_list[peer].numel():
                    out_list[peer].copy_(in_list[peer])
                continue
            if in_list[peer].numel():
                ops.append(dist.P2POp(dist.isend, in_list[peer], gpeer, self.group))
            if out_list[peer].numel():
                ops.append(dist.P2POp(dist.irecv, out_list[peer], gpeer, self.group))
        handle = _Works(dist.batch_isend_irecv(ops) if ops else [])
        if async_op:
            return handle
        handle.wait()
        return None

    def all_reduce_sum(self, t: torch.Tensor) -> torch.Tensor:
        self.dist.all_reduce(t, group=self.group)
        return t

    def barrier(self) -> None:
        """Stream-ordered: the current stream's later work on any rank runs after every
        rank's earlier work (a one-element all-reduce)."""
        if not hasattr(self, "_flag"):
            dev = self.device if self.device is not None else torch.cuda.current_device()
            self._flag = torch.zeros(1, dtype=torch.int32, device=dev)
        self.dist.all_reduce(self._flag, group=self.group)

    def peer_addresses(self, t: torch.Tensor) -> List[int]:
        """Every rank's t as this process addresses it: its own data_ptr, the others
        through the library's CUDA IPC mapping (handles all-gathered)."""
        h = torch.frombuffer(bytearray(L.moe_peer_export(t)), dtype=torch.uint8).to(t.device)
        hs = self.all_gather(h).cpu().numpy()
        return [t.data_ptr() if r == self.rank else L.moe_peer_import(hs[r].tobytes()) for r in range(self.world)]

    def release_peer(self, address: int) -> None:
        L.moe_peer_close(address)


# ----------------------------------------------------------------------------- host plan
def plan_rounds(kept: np.ndarray, world: int, cap: int):
    """Pack every destination's (source, expert) pieces into rounds of at most `cap`
    received rows.  kept [W, N]: rows source s keeps for expert e.  A destination
    takes its experts in order and, for each, the sources in order; a piece opens a
    new round when it does not fit the current one (a piece never exceeds T <= cap
    rows, since a token picks an expert at most once).  Returns (round_of [W, N], R):
    the round of each piece at its destination, and the number of rounds every rank
    runs (that of the busiest destination, at least 1).  Deterministic, so every
    rank computes the same plan."""
    W, N = kept.shape
    El = N // world
    round_of = np.zeros((W, N), np.int64)
    R = 1
    for d in range(world):
        cur, r = 0, 0
        for e in range(d * El, (d + 1) * El):
            for s in range(W):
                n = int(kept[s, e])
                if n > cap:
                    raise ValueError(f"a piece of {n} rows exceeds the receive capacity {cap}")
                if n and cur + n > cap:
                    r, cur = r + 1, 0
                round_of[s, e] = r
                cur += n
        R = max(R, r + 1)
    return round_of, R


@dataclass
class RoundPlan:
    offsets_all: np.ndarray        # [W, N + 1] offsets of the round's pieces only (moe_ep_plan input)
    send_start: List[int]          # per destination: first row of this rank's x_perm it sends
    send_count: List[int]          # per destination: rows sent
    recv_count: List[int]          # per source: rows received


def round_plans(offsets_all: np.ndarray, rank: int, world: int, cap: int) -> List[RoundPlan]:
    """The per-round exchange of rank `rank` (host side).  A source's pieces for one
    destination in one round cover a contiguous range of its experts (the round index
    never decreases along a destination's experts), hence a contiguous slice of its
    expert-ordered rows."""
    off = np.asarray(offsets_all, np.int64)
    W, N = off.shape[0], off.shape[1] - 1
    El = N // world
    kept = off[:, 1:] - off[:, :-1]
    round_of, R = plan_rounds(kept, world, cap)
    plans = []
    for r in range(R):
        kr = np.where(round_of == r, kept, 0)
        off_r = np.concatenate([np.zeros((W, 1), np.int64), np.cumsum(kr, axis=1)], axis=1)
        start, count = [], []
        for d in range(world):
            es = [e for e in range(d * El, (d + 1) * El) if round_of[rank, e] == r and kept[rank, e] > 0]
            start.append(int(off[rank, es[0]]) if es else 0)
            count.append(int(sum(kept[rank, e] for e in es)))
        recv = [int(kr[s, rank * El:(rank + 1) * El].sum()) for s in range(W)]
        plans.append(RoundPlan(off_r.astype(np.int32), start, count, recv))
    return plans


# ----------------------------------------------------------------------------- layer
class EPMoELayer:
    """Rank `rank` of `world`: routes its own T tokens over all N experts and computes
    the experts rank * N / W .. (rank + 1) * N / W - 1 for every rank's tokens.

    recv_factor: the receive buffer holds ceil(recv_factor * T * k) rows (at least T);
    1.0 is what a rank receives on average.  Skewed routing costs more rounds, never
    a failure.

    device_plan (peer exchange only): the receive buffer holds every row a rank can
    receive, W * T * min(k, N / W) (a token sends a rank at most one row per expert it
    picks there), so one round always suffices and the plan never leaves the device:
    a forward makes no host synchronisation (recv_factor is not used)."""

    def __init__(self, w: Workload, weights: dict, rank: int, world: int, device="cuda",
                 exchange=None, update_bias: bool = True, recv_factor: float = 1.0, peer: bool = False,
                 device_plan: bool = False):
        if w.N % world != 0:
            raise ValueError(f"{w.N} experts do not divide over {world} ranks")
        if w.fp8 or w.mxfp8 or w.nvfp4 or w.expert_choice or w.dtype != "bf16":
            raise ValueError("the expert-parallel layer runs bf16 token-choice routing")
        if not recv_factor > 0:
            raise ValueError("recv_factor must be positive")
        if device_plan and not peer:
            raise ValueError("the device-side plan needs the peer exchange")
        self.w, self.rank, self.world = w, rank, world
        self.El = w.N // world
        self.exchange = exchange
        dev = torch.device(device)
        self.dev = dev
        lo, hi = rank * self.El, (rank + 1) * self.El
        # the single-rank layer supplies routing, permutation, shared experts, combine, stats;
        # it keeps only this rank's experts
        local = {k: v for k, v in weights.items() if k not in ("w1", "w3", "w2")}
        self.base = MoELayer(w, local, dev, update_bias=False, gather_rows=False, fuse_shared=False)
        self.w1, self.w3, self.w2 = (weights[n][lo:hi].contiguous() for n in ("w1", "w3", "w2"))
        self.update_bias = update_bias and weights.get("bias") is not None
        self.peer = peer and world > 1
        self.device_plan = device_plan and self.peer
        if self.device_plan:
            self.recv_cap = max(world * w.T * min(w.k, self.El), 1)
        else:
            self.recv_cap = max(int(math.ceil(recv_factor * w.T * w.k)), w.T, 1)
        z = lambda *s, dtype=torch.bfloat16: torch.empty(s, dtype=dtype, device=dev)  # noqa: E731
        # two buffer sets (rounds alternate; one with the device-side plan): received rows
        # (later the results in arrival order), rows regrouped by local expert (later their
        # results), hidden rows; a single rank exchanges nothing and needs none
        nset = (1 if self.device_plan else 2) if world > 1 else 0
        # peer mode: the FFN runs in place on the receive buffer, and set 0 also holds
        # the shared expert's T rows after the routed ones when it rides in the same launches
        self.fuse_shared = (self.peer and self.base.fs > 0 and self.base.fs == w.f
                            and self.recv_cap + w.T < 2 ** 31)
        extra = w.T if self.fuse_shared else 0
        self.recv = [z(self.recv_cap + (extra if i == 0 else 0), w.d) for i in range(nset)]
        self.loc = [z(self.recv_cap, w.d) for _ in range(nset)] if not self.peer else []
        self.h_loc = [z(self.recv_cap + (extra if i == 0 else 0), w.f) for i in range(nset)]
        self.row_addr = z(w.T * w.k, dtype=torch.int64) if self.peer else None
        self.peer_rows: List[torch.Tensor] = []            # per buffer set: [W] addresses of every rank's set
        self._imported: List[int] = []
        # the regroup map is the NCCL exchange's (peer rows land in local-expert order)
        self.regroup_map = [z(0 if self.peer else self.recv_cap, dtype=torch.int32) for _ in range(nset)]
        self.local_offsets = [z(self.El + 1, dtype=torch.int32) for _ in range(nset)]
        self.send_splits = z(world, dtype=torch.int32)
        self.recv_splits = z(world, dtype=torch.int32)
        self.counts_global = z(w.N, dtype=torch.int32)
        self.plans: List[RoundPlan] = []

    # ---------------------------------------------------------------- phases
    def dispatch_prepare(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        """Route and permute this rank's tokens; returns the offsets to all-gather."""
        b, c = self.base, self.base.cfg
        b.route(x, stream)
        L.moe_permute(c, x, b.topk_idx, b.counts, b.offsets, b.row_of_slot, b.token_of_row, b.x_perm,
                      b.n_dropped, b.ws, stream)
        return b.offsets

    def plan(self, offsets_all: torch.Tensor, stream=None) -> int:
        """Plan the rounds from every rank's offsets (copied to the host: the one
        synchronisation) and upload every round's offsets at once.  Returns the
        number of rounds."""
        off = offsets_all.cpu().numpy()
        self.plans = round_plans(off, self.rank, self.world, self.recv_cap)
        stacked = np.stack([p.offsets_all for p in self.plans])
        host = torch.from_numpy(stacked).pin_memory() if self.dev.type == "cuda" else torch.from_numpy(stacked)
        self.round_offsets = host.to(self.dev, non_blocking=True)
        return len(self.plans)

    def round_begin(self, r: int, stream=None):
        """The device plan of round r (regroup map, local expert offsets) into buffer set r % 2."""
        i = r % 2
        L.moe_ep_plan(self.round_offsets[r], self.world, self.rank, self.send_splits, self.recv_splits,
                      self.local_offsets[i], self.regroup_map[i], stream)

    def send_slices(self, r: int) -> List[torch.Tensor]:
        p, x = self.plans[r], self.base.x_perm
        return [x[s:s + n] for s, n in zip(p.send_start, p.send_count)]

    def recv_slices(self, r: int) -> List[torch.Tensor]:
        """Per source, where its rows of round r land (source-major arrival order)."""
        p, buf = self.plans[r], self.recv[r % 2]
        q = np.concatenate([[0], np.cumsum(p.recv_count)]).astype(np.int64)
        return [buf[q[s]:q[s + 1]] for s in range(self.world)]

    def local_compute(self, r: int, stream=None):
        """Regroup round r's received rows by local expert, run the local experts'
        grouped FFN, and put the results back in arrival order (in the receive buffer)."""
        i, w = r % 2, self.w
        n_rows = self.local_offsets[i][self.El:]             # device scalar: rows received
        L.moe_rows_move(self.recv[i], self.regroup_map[i], n_rows, self.loc[i], scatter=True, stream=stream)
        L.moe_grouped_ffn(self.base.cfg, self.loc[i], self.recv_cap, self.local_offsets[i], self.El,
                          self.w1, self.w3, self.w2, w.f, self.h_loc[i], self.loc[i], stream)
        L.moe_rows_move(self.loc[i], self.regroup_map[i], n_rows, self.recv[i], scatter=False, stream=stream)

    def return_send_slices(self, r: int) -> List[torch.Tensor]:
        """Per source, the results of its rows (arrival order), to send back."""
        return self.recv_slices(r)

    def return_recv_slices(self, r: int) -> List[torch.Tensor]:
        """Per destination, where its results land in this rank's y_perm."""
        p, y = self.plans[r], self.base.y_perm
        return [y[s:s + n] for s, n in zip(p.send_start, p.send_count)]

    def stats_partial(self, stream=None) -> torch.Tensor:
        """This rank's sufficient statistics (fp64 [3N + 5]), to be summed over ranks."""
        b = self.base
        L.moe_router_stats_partial(b.cfg, b.counts, b.offsets, b.p_partial, b.lse, b.n_dropped, b.stats_part,
                                   margin=b.margin, stream=stream)
        return b.stats_part

    def finish(self, x: torch.Tensor, stream=None, partial_sum: Optional[torch.Tensor] = None,
               row_addr: Optional[torch.Tensor] = None, shared: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Shared experts, combine (base.y_perm holds the returned rows, or row_addr
        gives where each row's result is), statistics and bias update.  shared: the
        shared experts' output when already computed.  With partial_sum (the sum over
        ranks of stats_partial()) the statistics are the whole batch's and the bias
        update uses the summed counts; without it, this rank's statistics and no bias
        update."""
        b, c, w = self.base, self.base.cfg, self.w
        W = b.weights
        if shared is None and b.fs > 0:
            L.moe_grouped_ffn(c, x, w.T, b.shared_offsets, 1, W["ws1"], W["ws3"], W["ws2"], b.fs, b.hs, b.ys,
                              stream)
            shared = b.ys
        if row_addr is not None:
            L.moe_combine_peer(c, row_addr, b.row_of_slot, b.topk_w, shared, b.y, stream, shared_w=b.shared_w)
        else:
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
    def forward(self, x: torch.Tensor, stream=None, marks=None) -> torch.Tensor:
        """One layer forward with the real exchange.  `marks`, if given, is a list of 4
        CUDA events recorded on the compute stream: start, after route + permute, after
        the exchange and the local experts (all rounds), at the end."""
        ex = self.exchange
        comp = stream if stream is not None else torch.cuda.current_stream(self.dev)
        rec = (lambda i: marks[i].record(comp)) if marks is not None else (lambda i: None)
        rec(0)
        if self.world == 1:
            # nothing to exchange: every row stays, already grouped by expert
            b, w = self.base, self.w
            self.dispatch_prepare(x, comp)
            rec(1)
            L.moe_grouped_ffn(b.cfg, b.x_perm, w.T * w.k, b.offsets, self.El, self.w1, self.w3, self.w2, w.f,
                              b.h, b.y_perm, comp)
            rec(2)
            with torch.cuda.stream(comp):
                part = ex.all_reduce_sum(self.stats_partial(comp))
            y = self.finish(x, comp, part)
            rec(3)
            return y
        if self.peer:
            return self._forward_peer(x, comp, rec)
        self.dispatch_prepare(x, comp)
        rec(1)
        offsets_all = ex.all_gather(self.base.offsets)
        R = self.plan(offsets_all, comp)
        # collectives are issued from a side stream, so waiting for a transfer holds
        # back only the transfers queued behind it, never the expert compute
        if not hasattr(self, "_comm"):
            self._comm = torch.cuda.Stream(self.dev)
        comm = self._comm

        def dispatch(r):
            self.round_begin(r, comp)
            comm.wait_stream(comp)            # the plan and this round's rows are ready
            with torch.cuda.stream(comm):
                return ex.all_to_all(self.recv_slices(r), self.send_slices(r), async_op=True)

        back = []
        nxt = dispatch(0)
        for r in range(R):
            with torch.cuda.stream(comp):
                nxt.wait()                    # round r's rows have arrived
            if r + 1 < R:
                if r >= 1:
                    with torch.cuda.stream(comm):
                        back[r - 1].wait()    # buffer set (r + 1) % 2 is free once round r - 1 returned
                nxt = dispatch(r + 1)
            self.local_compute(r, comp)
            comm.wait_stream(comp)            # round r's results are ready
            with torch.cuda.stream(comm):
                back.append(ex.all_to_all(self.return_recv_slices(r), self.return_send_slices(r), async_op=True))
        with torch.cuda.stream(comp):
            for h in back:                    # every round's results are home
                h.wait()
        rec(2)
        with torch.cuda.stream(comp):
            part = ex.all_reduce_sum(self.stats_partial(comp))
        y = self.finish(x, comp, part)
        rec(3)
        return y

    # ---------------------------------------------------------------- one rank, peer memory
    def map_peers(self) -> None:
        """Every rank's receive buffers as this rank addresses them (collective: every
        rank calls it, at its first peer forward)."""
        if self.peer_rows:
            return
        for buf in self.recv:
            addrs = self.exchange.peer_addresses(buf)
            self._imported += [a for r, a in enumerate(addrs) if r != self.rank]
            self.peer_rows.append(torch.tensor(addrs, dtype=torch.int64).to(self.dev))

    def close(self) -> None:
        """Release the peer mappings (every rank; after the last forward has finished
        on every rank)."""
        for a in self._imported:
            self.exchange.release_peer(a)
        self._imported, self.peer_rows = [], []

    def _forward_peer(self, x: torch.Tensor, comp, rec) -> torch.Tensor:
        ex, b, c, w = self.exchange, self.base, self.base.cfg, self.w
        self.map_peers()
        with torch.cuda.stream(comp):
            b.route(x, comp)
            # the permutation without its row gather: the dispatch gathers from x
            L.moe_permute(c, x, b.topk_idx, b.counts, b.offsets, b.row_of_slot, b.token_of_row, None,
                          b.n_dropped, b.ws, comp)
            rec(1)
            offsets_all = ex.all_gather(b.offsets)
            if self.device_plan:
                # one round: its offsets are the gathered ones, on the device
                self.plans = []
                self.round_offsets = offsets_all.unsqueeze(0)
                R = 1
            else:
                R = self.plan(offsets_all, comp)
            n_rows = b.offsets[w.N:]
            shared = None
            Wt = b.weights
            for r in range(R):
                i = r % 2
                self.round_begin(r, comp)
                L.moe_ep_peer_plan(self.round_offsets[r], b.offsets, self.world, self.rank, self.peer_rows[i],
                                   w.d * 2, self.recv_cap, self.row_addr, comp)
                L.moe_ep_peer_dispatch(c, x, b.row_of_slot, self.row_addr, stream=comp)
                ex.barrier()                  # every rank's rows of round r have landed here
                if r == 0 and self.fuse_shared:
                    L.moe_grouped_ffn_shared(c, self.recv[0], self.recv_cap, self.local_offsets[0], self.El,
                                             self.w1, self.w3, self.w2, w.f, self.h_loc[0], self.recv[0], x, w.T,
                                             Wt["ws1"], Wt["ws3"], Wt["ws2"], comp)
                    shared = self.recv[0][self.recv_cap:self.recv_cap + w.T]
                else:
                    L.moe_grouped_ffn(c, self.recv[i], self.recv_cap, self.local_offsets[i], self.El, self.w1,
                                      self.w3, self.w2, w.f, self.h_loc[i], self.recv[i], comp)
                ex.barrier()                  # every rank's results of round r are ready
                if R > 1:
                    L.moe_ep_peer_collect(c, self.row_addr, n_rows, b.y_perm, stream=comp)
            rec(2)
            part = ex.all_reduce_sum(self.stats_partial(comp))
            y = self.finish(x, comp, part, row_addr=self.row_addr if R == 1 else None, shared=shared)
        rec(3)
        return y

    def rows_received(self) -> int:
        """Rows this rank's experts computed in the last forward (reads the device)."""
        if self.world == 1:
            return int(self.base.offsets[-1].item())
        if self.device_plan:
            return int(self.local_offsets[0][self.El].item())
        return sum(sum(p.recv_count) for p in self.plans)

    def kernel_launches(self, rounds: Optional[int] = None) -> int:
        # route, permute (4), combine, stats (2), bias; shared FFN (2)
        n = 1 + 4 + 1 + 2 + (1 if self.update_bias else 0)
        n += 2 if self.base.fs > 0 else 0
        if self.world == 1:
            return n + 2                                      # local FFN (2)
        R = (1 if self.device_plan else len(self.plans)) if rounds is None else rounds
        if self.peer:
            # permute without its gather (3); per round: two plans, dispatch, FFN (2), and
            # with several rounds a collect; the shared expert rides in round 0's FFN
            n -= 1
            n -= 2 if self.fuse_shared else 0
            return n + R * (1 + 1 + 1 + 2) + (R if R > 1 else 0)
        return n + R * (1 + 2 + 2)                            # per round: plan, two row moves, FFN (2)
