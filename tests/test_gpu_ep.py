"""Expert-parallel layer on one GPU.

* moe_ep_plan against the oracle's plan (integers, bit for bit);
* moe_rows_move against plain indexing;
* W = 2 and 4 ranks driven in lock step on one GPU, the all-to-alls done by the
  test with plain copies (no kernel of one rank waits for another): every rank's
  output equals the single-rank layer's on its tokens, bit for bit -- a row's
  expert result does not depend on which rows share its GEMM tile -- and the
  oracle's layer forward on its tokens within the bf16 bar; the router statistics,
  summed over ranks, equal the oracle's on the concatenated batch;
* one rank with a real NCCL exchange (world size 1).
"""
from __future__ import annotations

import os
import socket
from dataclasses import replace

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_21_b200 import _lib as L
from sparse_mixture_experts_21_b200.ep import EPMoELayer, TorchDistExchange
from sparse_mixture_experts_21_b200.layer import MoELayer
from sparse_mixture_experts_21_b200.synth import WORKLOADS, make_inputs
from tests.parity_util import (NEAR_TIE, TOL_BF16, TOL_STATS, expert_weights_fn, f64, i64, oracle_cfg, rel_err,
                               shared_weights)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("W,N", [(1, 8), (4, 16), (8, 256)])
def test_ep_plan_matches_oracle(W, N):
    rng = np.random.default_rng(W * N)
    kept = rng.integers(0, 40, size=(W, N))
    kept[:, 1] = 0                                          # an expert nobody routes to
    off = np.concatenate([np.zeros((W, 1), np.int64), np.cumsum(kept, axis=1)], axis=1).astype(np.int32)
    offsets_all = torch.tensor(off, device="cuda")
    El = N // W
    for rank in range(W):
        p = O.ep_plan(off, rank)
        cap = sum(p["recv"]) + 5
        send = torch.full((W,), -1, dtype=torch.int32, device="cuda")
        recv = torch.full((W,), -1, dtype=torch.int32, device="cuda")
        loc = torch.full((El + 1,), -1, dtype=torch.int32, device="cuda")
        rmap = torch.full((cap,), -7, dtype=torch.int32, device="cuda")
        L.moe_ep_plan(offsets_all, W, rank, send, recv, loc, rmap)
        torch.cuda.synchronize()
        assert send.cpu().tolist() == p["send"] and recv.cpu().tolist() == p["recv"]
        assert loc.cpu().numpy().tolist() == p["local_offsets"].tolist()
        R = sum(p["recv"])
        assert np.array_equal(rmap[:R].cpu().numpy(), p["regroup"])
        assert torch.all(rmap[R:] == -7)                   # entries past the total untouched


def test_rows_move_gather_and_scatter():
    g = torch.Generator(device="cuda").manual_seed(3)
    src = torch.randn(1000, 7168 // 8, generator=g, device="cuda").to(torch.bfloat16)
    perm = torch.randperm(1000, generator=g, device="cuda").to(torch.int32)
    n = torch.tensor([777], dtype=torch.int32, device="cuda")
    dst = torch.zeros_like(src)
    L.moe_rows_move(src, perm, n, dst, scatter=False)
    torch.cuda.synchronize()
    assert torch.equal(dst[:777], src[perm[:777].long()]) and torch.all(dst[777:] == 0)
    dst2 = torch.zeros_like(src)
    L.moe_rows_move(src, perm, None, dst2, scatter=True)
    torch.cuda.synchronize()
    want = torch.empty_like(src)
    want[perm.long()] = src
    assert torch.equal(dst2, want)


def _case(T=300):
    return replace(WORKLOADS["deepseek_v3"], name="v3_ep_small", T=T, d=256, N=32, k=4, f=256, n_groups=4,
                   topk_groups=2, n_shared=1, f_shared=256)


@pytest.mark.parametrize("W,recv_factor", [(2, 1.0), (4, 1.0), (4, 0.3)])
def test_ep_lock_step_matches_single_rank(W, recv_factor):
    w = _case()
    shared = make_inputs(w, "cuda", seed=0)                 # router, bias, experts: the same on every rank
    xs = [make_inputs(w, "cuda", seed=10 + r, experts=False)["x"] for r in range(W)]
    layers = [EPMoELayer(w, shared, r, W, "cuda", update_bias=False, recv_factor=recv_factor) for r in range(W)]
    # phase 1: route and permute; the offsets all-gather; every rank's plan
    offsets_all = torch.stack([lay.dispatch_prepare(x).clone() for lay, x in zip(layers, xs)])
    R = [lay.plan(offsets_all) for lay in layers]
    assert len(set(R)) == 1                                 # every rank runs the same rounds
    if recv_factor < 1.0:
        assert R[0] > 1
    for r in range(R[0]):
        for lay in layers:
            lay.round_begin(r)
        # the dispatch all-to-all, by copies: rank d receives from s what s sends to d
        for d in range(W):
            for s_ in range(W):
                layers[d].recv_slices(r)[s_].copy_(layers[s_].send_slices(r)[d])
        for lay in layers:
            lay.local_compute(r)
        # the return all-to-all
        for s_ in range(W):
            for d in range(W):
                layers[s_].return_recv_slices(r)[d].copy_(layers[d].return_send_slices(r)[s_])
    # the statistics all-reduce, by a sum
    psum = torch.stack([lay.stats_partial().clone() for lay in layers]).sum(0)
    ys = [lay.finish(x, partial_sum=psum) for lay, x in zip(layers, xs)]
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    cfg = oracle_cfg(w)
    for r in range(W):
        single = MoELayer(w, dict(shared, x=xs[r]), "cuda", update_bias=False)
        y_ref = single.forward(xs[r])
        torch.cuda.synchronize()
        assert torch.equal(ys[r][:w.T], y_ref[:w.T]), r
        assert torch.equal(layers[r].base.stats, layers[0].base.stats)     # global: the same on every rank
        # the oracle's forward on this rank's tokens (dropless: tokens are independent)
        out = O.layer_forward(f64(xs[r]), f64(shared["w_gate"]), cfg, expert_weights_fn(shared),
                              shared_weights(shared), bias=f64(shared["bias"]))
        clear = out["routing"]["margin"] >= NEAR_TIE
        assert clear.mean() > 0.95
        assert np.array_equal(i64(layers[r].base.topk_idx)[clear], out["routing"]["idx"][clear])
        assert rel_err(f64(ys[r][:w.T])[clear], out["y"][clear]) < TOL_BF16, r
    # global statistics against the oracle on the concatenated batch (counts and drops
    # from the GPU's expert choice, affinities and lse the oracle's own)
    x_all = torch.cat(xs)
    rall = O.route(f64(x_all), f64(shared["w_gate"]), cfg, bias=f64(shared["bias"]))
    idx_all = np.concatenate([i64(lay.base.topk_idx) for lay in layers])
    p = O.permutation(idx_all, w.N, None)
    ost = O.router_stats(p["counts"], p["kept"], rall["s"], rall["lse"], cfg, W * w.T, p["dropped_slots"],
                         p["dropped_tokens"], w.alpha, w.z_coef, f64(shared["bias"]))
    st = layers[0].base.stats_dict()
    for key in ("aux", "aux_raw", "z", "z_loss", "cv", "cv_kept", "bias_norm"):
        assert abs(st[key] - ost[key]) <= TOL_STATS * max(abs(ost[key]), 1e-30) + 1e-12, key
    assert st["T"] == W * w.T and st["R"] == p["R"] and st["dead"] == ost["dead"]
    assert torch.equal(layers[0].counts_global.cpu(), torch.tensor(p["counts"], dtype=torch.int32))
    assert rel_err(f64(layers[0].base.p_out), ost["P"]) < TOL_STATS


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_ep_one_rank_nccl():
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        w = _case(T=500)
        inp = make_inputs(w, "cuda", seed=0)
        bias0 = inp["bias"].clone()
        lay = EPMoELayer(w, inp, 0, 1, "cuda", exchange=TorchDistExchange(), update_bias=True)
        y = lay.forward(inp["x"])
        torch.cuda.synchronize()
        bias_ep = inp["bias"].clone()
        inp["bias"].copy_(bias0)
        single = MoELayer(w, inp, "cuda", update_bias=True)
        y_ref = single.forward(inp["x"])
        torch.cuda.synchronize()
        assert torch.equal(y[:w.T], y_ref[:w.T])
        assert torch.equal(bias_ep, inp["bias"])             # the same bias step
        assert L.moe_device_status() == L.MOE_OK
    finally:
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- forward() with rounds, W threads
class _Hub:
    """Meeting point of W in-process ranks: a barrier and one slot per rank."""

    def __init__(self, world):
        import threading
        self.world = world
        self.barrier = threading.Barrier(world, timeout=120)
        self.slot = [None] * world


class _ThreadExchange:
    """The exchange interface of EPMoELayer for W ranks run as threads on one GPU.
    Data moves by device copies on the receiving rank's current stream, ordered after
    the sender's data by CUDA events recorded before a host barrier; no kernel waits
    for another rank's kernel."""

    def __init__(self, hub, rank):
        self.hub, self.rank, self.world = hub, rank, hub.world

    def _post(self, item):
        ev = torch.cuda.Event()
        ev.record()
        self.hub.barrier.wait()
        self.hub.slot[self.rank] = (item, ev)
        self.hub.barrier.wait()
        got = list(self.hub.slot)
        self.hub.barrier.wait()
        for _, e in got:
            torch.cuda.current_stream().wait_event(e)
        return [g[0] for g in got]

    def all_gather(self, t):
        return torch.stack([x.clone() for x in self._post(t)])

    def all_to_all(self, out_list, in_list, async_op=False):
        ins = self._post(list(in_list))
        for s in range(self.world):
            out_list[s].copy_(ins[s][self.rank])
        arrived = torch.cuda.Event()
        arrived.record()
        self._post(None)                               # senders may reuse their buffers after this

        class _H:
            def wait(self_inner):                      # the caller's stream waits for the data
                torch.cuda.current_stream().wait_event(arrived)
        if async_op:
            return _H()
        _H().wait()
        return None

    def all_reduce_sum(self, t):
        parts = self._post(t)
        total = torch.stack([p.clone() for p in parts]).sum(0)
        self._post(None)
        t.copy_(total)
        return t


@pytest.mark.parametrize("W,recv_factor", [(2, 0.4), (4, 1.0)])
def test_ep_forward_threads_matches_single_rank(W, recv_factor):
    """EPMoELayer.forward (rounds on two buffer sets, collectives from a side stream)
    for W ranks run as threads on one GPU: each rank's output equals the single-rank
    layer's on its tokens, and the bias update uses the counts of all ranks."""
    import threading
    w = _case()
    shared = make_inputs(w, "cuda", seed=0)
    xs = [make_inputs(w, "cuda", seed=30 + r, experts=False)["x"] for r in range(W)]
    bias0 = shared["bias"].clone()
    hub = _Hub(W)
    weights = [dict(shared, bias=bias0.clone()) for _ in range(W)]
    layers = [EPMoELayer(w, weights[r], r, W, "cuda", exchange=_ThreadExchange(hub, r), update_bias=True,
                         recv_factor=recv_factor) for r in range(W)]
    ys, errs = [None] * W, []

    def run(r):
        try:
            with torch.cuda.stream(torch.cuda.Stream()):
                ys[r] = layers[r].forward(xs[r]).clone()
                torch.cuda.current_stream().synchronize()
        except Exception as e:          # reported below
            errs.append(e)
            hub.barrier.abort()

    th = [threading.Thread(target=run, args=(r,)) for r in range(W)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errs, errs
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    if recv_factor < 1.0:
        assert len(layers[0].plans) > 1
    counts = torch.zeros(w.N, dtype=torch.int64, device="cuda")
    for r in range(W):
        single = MoELayer(w, dict(shared, x=xs[r], bias=bias0.clone()), "cuda", update_bias=False)
        y_ref = single.forward(xs[r])
        torch.cuda.synchronize()
        assert torch.equal(ys[r][:w.T], y_ref[:w.T]), r
        counts += single.counts.long()
    ref_bias = O.bias_update(f64(bias0), counts.cpu().numpy(), rate=w.bias_rate)
    for r in range(W):
        assert np.max(np.abs(f64(weights[r]["bias"]) - ref_bias)) < 1e-7
