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


@pytest.mark.parametrize("W", [2, 4])
def test_ep_lock_step_matches_single_rank(W):
    w = _case()
    shared = make_inputs(w, "cuda", seed=0)                 # router, bias, experts: the same on every rank
    xs = [make_inputs(w, "cuda", seed=10 + r, experts=False)["x"] for r in range(W)]
    layers = [EPMoELayer(w, shared, r, W, "cuda", update_bias=False) for r in range(W)]
    # phase 1: route and permute; the offsets all-gather
    offsets_all = torch.stack([lay.dispatch_prepare(x).clone() for lay, x in zip(layers, xs)])
    plans = [lay.plan(offsets_all) for lay in layers]
    send = [p[0] for p in plans]
    recv = [p[1] for p in plans]
    # the dispatch all-to-all, by copies: rank d receives from s the rows s sends to d
    for d in range(W):
        q = 0
        for s in range(W):
            start = sum(send[s][:d])
            n = send[s][d]
            layers[d].recv_x[q:q + n] = layers[s].base.x_perm[start:start + n]
            q += n
    for lay in layers:
        lay.local_compute()
    # the return all-to-all
    for s in range(W):
        for d in range(W):
            off_in_d = sum(recv[d][:s])                     # where s's rows sit among d's arrivals
            start, n = sum(send[s][:d]), send[s][d]
            layers[s].base.y_perm[start:start + n] = layers[d].recv_y[off_in_d:off_in_d + n]
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
