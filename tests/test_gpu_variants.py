"""GPU-vs-oracle parity of the routing variants, through the C ABI:
non-renormalised weights, the shared-expert sink, the moving-average bias
controller and the per-sequence (length-normalised) bias update."""
from __future__ import annotations

from dataclasses import replace

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_21_b200 import _lib as L
from sparse_mixture_experts_21_b200.layer import MoELayer, make_config
from sparse_mixture_experts_21_b200.synth import WORKLOADS, make_inputs, random_routing
from tests.parity_util import (NEAR_TIE, expert_weights_fn, f64, i64, oracle_cfg, rel_err,
                               shared_weights, tol_for)

pytestmark = pytest.mark.gpu

DS_SMALL = replace(WORKLOADS["deepseekmoe_16b"], name="dsmoe_small", T=777, d=264, N=16, f=192,
                   f_shared=192)


def _run(w):
    inp = make_inputs(w, "cuda")
    lay = MoELayer(w, inp, "cuda", update_bias=False)
    lay.forward(inp["x"])
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    return lay, inp


@pytest.mark.parametrize("score", ["softmax", "sigmoid"])
def test_renorm_off(score):
    w = replace(DS_SMALL, renorm=False, score=score)
    lay, inp = _run(w)
    r = O.route(f64(inp["x"]), f64(inp["w_gate"]), oracle_cfg(w))
    clear = r["margin"] >= NEAR_TIE
    assert np.array_equal(i64(lay.topk_idx)[clear], r["idx"][clear])
    assert np.max(np.abs(f64(lay.topk_w)[clear] - r["w"][clear])) < 2e-5
    wts = O.gate_weights(r["s"], i64(lay.topk_idx), False)
    out = O.layer_forward(f64(inp["x"]), None, oracle_cfg(w), expert_weights_fn(inp), shared_weights(inp),
                          routing={"idx": i64(lay.topk_idx), "w": wts})
    assert rel_err(f64(lay.y[:w.T]), out["y"]) < tol_for(w)


@pytest.mark.parametrize("score,N,dtype", [("softmax", 16, "bf16"), ("sigmoid", 64, "bf16"),
                                           ("sigmoid", 300, "bf16"), ("softmax", 8, "fp32")])
def test_shared_expert_sink(score, N, dtype):
    """N + 1 <= 256 runs the tensor-core router, 301 gate rows and fp32 the FMA one."""
    d = 128 if dtype == "fp32" else 264
    w = replace(DS_SMALL, score=score, N=N, n_shared=1, shared_sink=True, dtype=dtype, d=d,
                k=2 if N == 8 else 6)
    lay, inp = _run(w)
    cfg = oracle_cfg(w)
    r = O.route_shared_sink(f64(inp["x"]), f64(inp["w_gate"]), cfg)
    clear = r["margin"] >= NEAR_TIE
    assert np.array_equal(i64(lay.topk_idx)[clear], r["idx"][clear])
    assert np.max(np.abs(f64(lay.topk_w)[clear] - r["w"][clear])) < 2e-5
    assert np.max(np.abs(f64(lay.shared_w[:w.T])[clear] - r["w_shared"][clear])) < 2e-5
    assert np.allclose(f64(lay.topk_w).sum(1) + f64(lay.shared_w[:w.T]), 1.0, atol=1e-5)
    assert rel_err(f64(lay.lse), r["lse"]) < 1e-5
    # whole layer, oracle fed the GPU's expert choice
    sel = np.take_along_axis(r["s"], i64(lay.topk_idx), 1)
    den = sel.sum(1) + r["s_shared"]
    out = O.layer_forward(f64(inp["x"]), None, cfg, expert_weights_fn(inp), None,
                          routing={"idx": i64(lay.topk_idx), "w": sel / den[:, None]})
    y_ref = out["y"] + (r["s_shared"] / den)[:, None] * O.swiglu_ffn(f64(inp["x"]), *shared_weights(inp))
    assert rel_err(f64(lay.y[:w.T]), y_ref) < tol_for(w)


def test_bias_update_ema_steps():
    w = WORKLOADS["deepseek_v3"]
    c = make_config(w)
    rng = np.random.default_rng(3)
    b0 = rng.normal(scale=0.05, size=w.N).astype(np.float32)
    bias = torch.tensor(b0, device="cuda")
    ema = torch.zeros(w.N, device="cuda")
    b_ref, e_ref = b0.astype(np.float64), np.zeros(w.N)
    for step in range(4):
        counts = rng.integers(0, 2000, size=w.N).astype(np.int32)
        L.moe_bias_update_ema(c, torch.tensor(counts, device="cuda"), ema, 0.8, bias, 1e-3, 0.0)
        b_ref, e_ref = O.bias_update_ema(b_ref, counts, e_ref, 0.8, 1e-3)
    torch.cuda.synchronize()
    assert np.max(np.abs(f64(ema) - e_ref)) <= 1e-6 * np.max(np.abs(e_ref))
    assert np.max(np.abs(f64(bias) - b_ref)) < 1e-7


def test_bias_update_seq():
    w = WORKLOADS["deepseek_v3"]
    T, N, k = 5000, w.N, w.k
    c = make_config(w, T=T)
    rng = np.random.default_rng(4)
    cuts = np.sort(rng.choice(np.arange(1, T), size=11, replace=False))
    off = np.concatenate([[0], cuts, [T]]).astype(np.int32)
    off[5] = off[4]                                         # one empty sequence
    idx = random_routing(T, N, k, "cuda", seed=9)
    bias = torch.zeros(N, device="cuda")
    ws = torch.empty(8 * (len(off) - 1) * N, dtype=torch.uint8, device="cuda")
    L.moe_bias_update_seq(c, idx, torch.tensor(off, device="cuda"), len(off) - 1, bias, 1e-3, 0.0, ws)
    torch.cuda.synchronize()
    load = O.sequence_load(i64(idx), off, N)
    ref = O.bias_update_from_load(np.zeros(N), load, 1e-3)
    assert np.array_equal(f64(bias) != 0, ref != 0)
    assert np.max(np.abs(f64(bias) - ref)) < 1e-9


# ----------------------------------------------------------------------------- expert choice
def ec_capacity(w):
    return L.expert_choice_capacity(make_config(w))


@pytest.mark.parametrize("score,dtype", [("softmax", "bf16"), ("sigmoid", "bf16"), ("softmax", "fp32")])
def test_expert_choice_layer(score, dtype):
    d = 128 if dtype == "fp32" else 264
    w = replace(DS_SMALL, score=score, dtype=dtype, d=d, expert_choice=True)
    lay, inp = _run(w)
    C = ec_capacity(w)
    cfg = oracle_cfg(w)
    s_ref = O.affinity(O.router_logits(f64(inp["x"]), f64(inp["w_gate"])), cfg.score_fn)
    s_gpu = f64(lay.scores).T                                   # [T, N]
    assert np.max(np.abs(s_gpu - s_ref)) < 1e-5
    # the selection, decided on the GPU's own fp32 scores on both sides
    ec = O.expert_choice(s_gpu, C)
    assert np.array_equal(i64(lay.row_of), ec["row_of"])
    assert np.array_equal(i64(lay.token_of_row)[: w.N * C], ec["token_of_row"])
    assert np.array_equal(i64(lay.offsets), ec["offsets"])
    assert int(lay.n_unpicked.item()) == ec["unpicked"]
    # expert rows and the combine against the oracle (fp64 affinities, same selection)
    off = ec["offsets"]
    get = expert_weights_fn(inp)
    y_rows = np.zeros((w.N * C, w.d))
    for e in range(w.N):
        y_rows[off[e]:off[e + 1]] = O.swiglu_ffn(f64(inp["x"])[ec["token_of_row"][off[e]:off[e + 1]]], *get(e))
    assert rel_err(f64(lay.y_perm[: w.N * C]), y_rows) < tol_for(w)
    ys = O.swiglu_ffn(f64(inp["x"]), *shared_weights(inp))
    y_ref = O.expert_choice_combine(y_rows, ec["row_of"], s_ref, ys)
    assert rel_err(f64(lay.y[:w.T]), y_ref) < tol_for(w)


def test_expert_choice_ties_and_capacity_edges():
    """Quantised scores with many exact ties; C = 1 and C = T."""
    w = replace(DS_SMALL, T=700, N=12, expert_choice=True)
    c = make_config(w)
    rng = np.random.default_rng(11)
    s = (rng.integers(0, 5, size=(w.T, w.N)) / 8.0).astype(np.float32)
    scores = torch.tensor(s.T.copy(), device="cuda")
    x = torch.randn(w.T, w.d, device="cuda").to(torch.bfloat16)
    for C in (1, 37, w.T):
        row_of = torch.empty(w.N, w.T, dtype=torch.int32, device="cuda")
        tor = torch.empty(w.N * C, dtype=torch.int32, device="cuda")
        off = torch.empty(w.N + 1, dtype=torch.int32, device="cuda")
        xp = torch.empty(w.N * C, w.d, dtype=torch.bfloat16, device="cuda")
        L.moe_expert_choice(c, x, scores, C, row_of, tor, off, xp)
        torch.cuda.synchronize()
        ec = O.expert_choice(s.astype(np.float64), C)
        assert np.array_equal(i64(row_of), ec["row_of"]) and np.array_equal(i64(tor), ec["token_of_row"])
        assert torch.equal(xp, x[tor.long()])


def test_expert_choice_full_size():
    """The DeepSeekMoE-16B-shaped expert-choice workload (T = 8192, 64 experts, C = 768):
    the selection bit for bit on the GPU's own affinities, sampled expert rows, and the
    combine on sampled tokens."""
    w = WORKLOADS["ec_deepseekmoe_16b"]
    lay, inp = _run(w)
    C = ec_capacity(w)
    assert C == 768
    s_gpu = f64(lay.scores).T                                   # [T, N]
    ec = O.expert_choice(s_gpu, C)
    assert np.array_equal(i64(lay.row_of), ec["row_of"])
    assert np.array_equal(i64(lay.token_of_row)[: w.N * C], ec["token_of_row"])
    assert int(lay.n_unpicked.item()) == ec["unpicked"]
    rng = np.random.default_rng(5)
    get = expert_weights_fn(inp)
    x64 = f64(inp["x"])
    for e in rng.choice(w.N, size=4, replace=False):
        rows = np.sort(rng.choice(C, size=24, replace=False)) + e * C
        toks = ec["token_of_row"][rows]
        ref = O.swiglu_ffn(x64[toks], *get(int(e)))
        assert rel_err(f64(lay.y_perm[torch.tensor(rows, device="cuda")]), ref) < tol_for(w)
    # combine on sampled tokens: shared experts + picked experts weighted by their affinity
    tok = np.sort(rng.choice(w.T, size=16, replace=False))
    ys = O.swiglu_ffn(x64[tok], *shared_weights(inp))
    # the GPU's expert rows (checked above by sampling) fed to the oracle's combine
    y_rows = np.zeros((w.N * C, w.d))
    ro = ec["row_of"]                                           # [N, T]: row of (expert, token) or -1
    need = sorted({int(ro[e, t]) for t in tok for e in range(w.N) if ro[e, t] >= 0})
    y_rows[need] = f64(lay.y_perm[torch.tensor(need, device="cuda")])
    y_ref = np.stack([ys[i] + sum(s_gpu[t, e] * y_rows[ro[e, t]] for e in range(w.N) if ro[e, t] >= 0)
                      for i, t in enumerate(tok)])
    assert rel_err(f64(lay.y[torch.tensor(tok, device="cuda")]), y_ref) < tol_for(w)
