"""GPU-vs-oracle parity of every step of the layer, through the C ABI.

Reduced shapes of each workload family span several tiles and ragged tails and
are checked element by element; the full-size workloads are checked on sampled
tokens and rows plus every integer output.  Integer outputs (indices, counts,
offsets, row maps, drops) must be bit-exact; floating outputs within
max|a-b|/max|b| <= 2e-2 (bf16) or 1e-4 (fp32), statistics within 1e-5.  Tokens
whose k-th vs (k+1)-th selection margin is below 1e-4 are excluded from the
index comparison and counted; the permutation is cross-fed (the oracle permutes
the GPU's routing) so that one near-tie cannot cascade.
"""
from __future__ import annotations

from dataclasses import replace

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_21_b200 import _lib as L
from sparse_mixture_experts_21_b200.layer import MoELayer, make_config
from sparse_mixture_experts_21_b200.synth import WORKLOADS, make_inputs, random_routing, torch_dtype
from tests.parity_util import (NEAR_TIE, TOL_STATS, expert_weights_fn, f64, i64, oracle_cfg,
                               rel_err, shared_weights, tol_for)

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny_top2_fp32": WORKLOADS["tiny_top2_fp32"],
    "mixtral_small": replace(WORKLOADS["mixtral_8x7b"], name="mixtral_small", T=513, d=512, f=1024),
    "dsmoe_small": replace(WORKLOADS["deepseekmoe_16b"], name="dsmoe_small", T=777, d=264, N=16,
                           f=192, f_shared=192),
    "v3_small": replace(WORKLOADS["deepseek_v3"], name="v3_small", T=1000, d=512, N=64, f=256,
                        f_shared=256),
    "switch_small": replace(WORKLOADS["switch_skewed"], name="switch_small", T=2000, d=256, N=32,
                            f=512),
}


def _run(w, seed=0, update_bias=False):
    torch.cuda.synchronize()
    inp = make_inputs(w, "cuda", seed=seed)
    bias0 = None if inp["bias"] is None else inp["bias"].clone()
    lay = MoELayer(w, inp, "cuda", update_bias=update_bias)
    lay.forward(inp["x"])
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    return lay, inp, bias0


@pytest.fixture(scope="module")
def small_runs():
    return {name: _run(w) for name, w in SMALL.items()}


# ----------------------------------------------------------------------------- routing
def _check_route(w, lay, inp, tokens):
    cfg = oracle_cfg(w)
    x = f64(inp["x"])[tokens]
    r = O.route(x, f64(inp["w_gate"]), cfg, bias=f64(inp["bias"]), logit_offset=f64(inp["logit_offset"]))
    gidx = i64(lay.topk_idx)[tokens]
    gw = f64(lay.topk_w)[tokens]
    clear = r["margin"] >= NEAR_TIE
    n_tie = int((~clear).sum())
    assert np.array_equal(gidx[clear], r["idx"][clear]), "expert indices differ on a clear token"
    assert np.max(np.abs(gw[clear] - r["w"][clear])) < 2e-5
    assert rel_err(f64(lay.lse)[tokens], r["lse"]) < 1e-5
    gm = f64(lay.margin)[tokens]
    fin = np.isfinite(r["margin"]) & clear
    assert np.all(np.abs(gm[fin] - r["margin"][fin]) < 1e-4 + 1e-4 * np.abs(r["margin"][fin]))
    return n_tie, r


@pytest.mark.parametrize("name", list(SMALL))
def test_route_parity(small_runs, name):
    lay, inp, _ = small_runs[name]
    w = SMALL[name]
    n_tie, r = _check_route(w, lay, inp, np.arange(w.T))
    print(f"{name}: near-ties {n_tie}/{w.T}")
    # weights sum to one, k distinct experts
    assert np.allclose(f64(lay.topk_w).sum(1), 1.0, atol=1e-5)
    gidx = i64(lay.topk_idx)
    assert all(len(set(row)) == w.k for row in gidx.tolist())


# ----------------------------------------------------------------------------- permutation
def _check_permute(w, lay, inp):
    idx = i64(lay.topk_idx)
    p = O.permutation(idx, w.N, O.capacity(oracle_cfg(w), w.T))
    assert np.array_equal(i64(lay.counts), p["counts"])
    assert np.array_equal(i64(lay.offsets), p["offsets"])
    assert np.array_equal(i64(lay.row_of_slot), p["row_of_slot"])
    R = p["R"]
    assert np.array_equal(i64(lay.token_of_row)[:R], p["token_of_row"])
    assert i64(lay.n_dropped).tolist() == [p["dropped_slots"], p["dropped_tokens"]]
    # the gather is a byte copy (layers whose grouped FFN reads x itself write none)
    if lay.x_perm is not None:
        tor = lay.token_of_row[:R].long()
        assert torch.equal(lay.x_perm[:R], inp["x"][tor])
    return p


@pytest.mark.parametrize("name", list(SMALL))
def test_permute_parity(small_runs, name):
    lay, inp, _ = small_runs[name]
    p = _check_permute(SMALL[name], lay, inp)
    if SMALL[name].capacity != "dropless":
        assert p["dropped_slots"] > 0


# ----------------------------------------------------------------------------- expert FFN
def _check_ffn_rows(w, lay, inp, rows_by_expert):
    get = expert_weights_fn(inp)
    xs, hs, ys, hr, yr = [], [], [], [], []
    for e, rows in rows_by_expert.items():
        if len(rows) == 0:
            continue
        xr = f64(inp["x"][lay.token_of_row[rows].long()])
        w1, w3, w2 = get(e)
        hr.append(O.swiglu_hidden(xr, w1, w3))
        yr.append(O.swiglu_ffn(xr, w1, w3, w2))
        hs.append(f64(lay.h[rows]))
        ys.append(f64(lay.y_perm[rows]))
    tol = tol_for(w)
    assert rel_err(np.concatenate(hs), np.concatenate(hr)) < tol
    assert rel_err(np.concatenate(ys), np.concatenate(yr)) < tol


@pytest.mark.parametrize("name", list(SMALL))
def test_grouped_ffn_parity(small_runs, name):
    lay, inp, _ = small_runs[name]
    w = SMALL[name]
    off = i64(lay.offsets)
    _check_ffn_rows(w, lay, inp, {e: torch.arange(off[e], off[e + 1], device="cuda") for e in range(w.N)})


@pytest.mark.parametrize("name", [n for n in SMALL if SMALL[n].n_shared > 0])
def test_shared_ffn_parity(small_runs, name):
    lay, inp, _ = small_runs[name]
    w = SMALL[name]
    ref = O.swiglu_ffn(f64(inp["x"]), *shared_weights(inp))
    assert rel_err(f64(lay.ys[:w.T]), ref) < tol_for(w)


# ----------------------------------------------------------------------------- combine
@pytest.mark.parametrize("name", list(SMALL))
def test_combine_parity(small_runs, name):
    lay, inp, _ = small_runs[name]
    w = SMALL[name]
    ys = f64(lay.ys[:w.T]) if lay.fs > 0 else None
    ref = O.combine(f64(lay.y_perm), i64(lay.row_of_slot), f64(lay.topk_w), ys, w.T, w.d)
    assert rel_err(f64(lay.y[:w.T]), ref) < tol_for(w)


# ----------------------------------------------------------------------------- whole layer
@pytest.mark.parametrize("name", list(SMALL))
def test_layer_end_to_end(small_runs, name):
    """The layer output against the oracle's own forward (its own routing)."""
    lay, inp, _ = small_runs[name]
    w = SMALL[name]
    cfg = oracle_cfg(w)
    out = O.layer_forward(f64(inp["x"]), f64(inp["w_gate"]), cfg, expert_weights_fn(inp),
                          shared_weights(inp), bias=f64(inp["bias"]),
                          logit_offset=f64(inp["logit_offset"]), alpha=w.alpha, z_coef=w.z_coef)
    margin = out["routing"]["margin"]
    clear = margin >= NEAR_TIE
    if np.all(clear):
        assert rel_err(f64(lay.y[:w.T]), out["y"]) < tol_for(w)
        st, ost = lay.stats_dict(), out["stats"]
        for key in ("aux", "aux_raw", "z", "cv", "cv_kept"):
            assert abs(st[key] - ost[key]) <= TOL_STATS * max(abs(ost[key]), 1e-30), key
        for key in ("dead", "dropped_slots", "dropped_tokens"):
            assert st[key] == ost[key], key
    elif w.capacity == "dropless":
        # tokens are independent when nothing is dropped: compare the clear ones
        assert rel_err(f64(lay.y[:w.T])[clear], out["y"][clear]) < tol_for(w)
    else:
        # a near-tie can move a capacity cut: feed the oracle the GPU's expert choice
        wts = O.gate_weights(out["routing"]["s"], i64(lay.topk_idx), w.renorm)
        out2 = O.layer_forward(f64(inp["x"]), None, cfg, expert_weights_fn(inp), shared_weights(inp),
                               routing={"idx": i64(lay.topk_idx), "w": wts})
        assert rel_err(f64(lay.y[:w.T]), out2["y"]) < tol_for(w)


@pytest.mark.parametrize("name", list(SMALL))
def test_stats_parity(small_runs, name):
    """Statistics against the oracle, fed the GPU's integer routing decision."""
    lay, inp, _ = small_runs[name]
    w = SMALL[name]
    cfg = oracle_cfg(w)
    r = O.route(f64(inp["x"]), f64(inp["w_gate"]), cfg, bias=f64(inp["bias"]),
                logit_offset=f64(inp["logit_offset"]))
    p = O.permutation(i64(lay.topk_idx), w.N, O.capacity(cfg, w.T))
    ost = O.router_stats(p["counts"], p["kept"], r["s"], r["lse"], cfg, w.T, p["dropped_slots"],
                         p["dropped_tokens"], w.alpha, w.z_coef, f64(inp["bias"]))
    st = lay.stats_dict()
    for key in ("aux", "aux_raw", "z", "z_loss", "cv", "cv_kept", "bias_norm"):
        assert abs(st[key] - ost[key]) <= TOL_STATS * max(abs(ost[key]), 1e-30) + 1e-12, key
    for key in ("dead", "dropped_slots", "dropped_tokens"):
        assert st[key] == ost[key], key
    assert st["R"] == p["R"] and st["T"] == w.T
    assert rel_err(f64(lay.f_out), ost["f"]) < TOL_STATS
    assert rel_err(f64(lay.p_out), ost["P"]) < TOL_STATS
    _check_near_ties(st, lay, r["margin"])


def _check_near_ties(st, lay, oracle_margin, max_frac=0.05):
    """The reported near-tie count is the number of the GPU's margins below the
    threshold, it agrees with the oracle's count up to tokens whose margin sits within
    a factor 2 of the threshold (where fp32 and fp64 may fall on different sides),
    and near-ties stay a small fraction of the tokens."""
    gm = f64(lay.margin)[:len(oracle_margin)]
    assert st["near_ties"] == int((gm < NEAR_TIE).sum())
    n_oracle = int((oracle_margin < NEAR_TIE).sum())
    border = int(((oracle_margin >= NEAR_TIE / 2) & (oracle_margin < 2 * NEAR_TIE)).sum())
    assert abs(st["near_ties"] - n_oracle) <= border
    assert n_oracle <= max_frac * len(oracle_margin)
    return n_oracle


def test_bias_update_parity():
    w = SMALL["v3_small"]
    lay, inp, b0 = _run(w, update_bias=True)
    ref = O.bias_update(f64(b0), i64(lay.counts), rate=w.bias_rate)
    assert np.max(np.abs(f64(inp["bias"]) - ref)) < 1e-7
    # clamp variant through the C ABI
    b = torch.full((w.N,), 0.0095, device="cuda")
    L.moe_bias_update(make_config(w), lay.counts, b, 1e-3, 1e-2)
    torch.cuda.synchronize()
    refc = O.bias_update(np.full(w.N, 0.0095, dtype=np.float32).astype(np.float64), i64(lay.counts),
                         rate=1e-3, clamp=1e-2)
    assert np.max(np.abs(f64(b) - refc)) < 1e-7


def test_deterministic_twice():
    w = SMALL["dsmoe_small"]
    inp = make_inputs(w, "cuda")
    lay = MoELayer(w, inp, "cuda", update_bias=False)
    lay.forward(inp["x"])
    first = [t.clone() for t in (lay.topk_idx, lay.topk_w, lay.row_of_slot, lay.token_of_row, lay.y_perm,
                                 lay.y, lay.stats)]
    lay.forward(inp["x"])
    torch.cuda.synchronize()
    second = (lay.topk_idx, lay.topk_w, lay.row_of_slot, lay.token_of_row, lay.y_perm, lay.y, lay.stats)
    for a, b in zip(first, second):
        assert torch.equal(a, b)


# ----------------------------------------------------------------------------- edge cases
@pytest.mark.parametrize("T", [1, 31, 257])
def test_ragged_token_counts(T):
    w = replace(SMALL["v3_small"], T=T)
    lay, inp, _ = _run(w)
    _check_route(w, lay, inp, np.arange(T))
    _check_permute(w, lay, inp)
    off = i64(lay.offsets)
    _check_ffn_rows(w, lay, inp, {e: torch.arange(off[e], off[e + 1], device="cuda") for e in range(w.N)})


def test_k_equals_n():
    w = replace(SMALL["mixtral_small"], T=100, N=4, k=4)
    lay, inp, _ = _run(w)
    _check_permute(w, lay, inp)
    out = O.layer_forward(f64(inp["x"]), f64(inp["w_gate"]), oracle_cfg(w), expert_weights_fn(inp))
    assert rel_err(f64(lay.y[:w.T]), out["y"]) < tol_for(w)


def _permute_with(w, idx):
    """Run moe_permute on a given routing (device) and compare with the oracle."""
    c = make_config(w)
    T, k, N = w.T, w.k, w.N
    x = torch.randn(T, w.d, device="cuda").to(torch_dtype(w))
    dev = lambda *s, dtype=torch.int32: torch.full(s, -7, dtype=dtype, device="cuda")  # noqa: E731
    counts, offsets, ros, tor, nd = dev(N), dev(N + 1), dev(T, k), dev(T * k), dev(2)
    xp = torch.zeros(T * k, w.d, dtype=torch_dtype(w), device="cuda")
    ws = torch.empty(max(L.workspace_size(c), 16), dtype=torch.uint8, device="cuda")
    L.moe_permute(c, x, idx, counts, offsets, ros, tor, xp, nd, ws)
    torch.cuda.synchronize()
    p = O.permutation(i64(idx), N, O.capacity(oracle_cfg(w), T))
    assert np.array_equal(i64(counts), p["counts"]) and np.array_equal(i64(offsets), p["offsets"])
    assert np.array_equal(i64(ros), p["row_of_slot"])
    assert np.array_equal(i64(tor)[:p["R"]], p["token_of_row"])
    assert i64(nd).tolist() == [p["dropped_slots"], p["dropped_tokens"]]
    assert torch.equal(xp[:p["R"]], x[tor[:p["R"]].long()])
    return p


def test_permute_all_tokens_to_one_expert_with_capacity():
    w = replace(SMALL["switch_small"], T=3000, N=16, k=2, capacity="ceil_cf_T_over_N", cf=1.0)
    idx = random_routing(w.T, w.N, w.k, "cuda", seed=3, hot=5)
    p = _permute_with(w, idx)
    assert p["kept"][5] == -(-w.T // w.N) and p["dropped_slots"] > 0


def test_permute_floor_capacity_variant_and_empty_experts():
    w = replace(SMALL["dsmoe_small"], T=600, N=64, k=2, capacity="floor_cf_k_T_over_N", cf=0.5)
    idx = random_routing(w.T, 8, w.k, "cuda", seed=4)          # only experts 0..7 used
    p = _permute_with(w, idx)
    assert (p["counts"][8:] == 0).all() and p["dropped_slots"] > 0


def test_permute_many_blocks_dropless():
    w = replace(SMALL["v3_small"], T=5000, N=256, k=8)
    idx = random_routing(w.T, w.N, w.k, "cuda", seed=5)
    _permute_with(w, idx)


def test_permute_invalid_expert_ids_are_dropped_and_flagged():
    """Expert ids outside [0, N) and repeats within a token: those slots are treated
    as dropped (row -1) and never dereferenced, the rest is the oracle's permutation
    of the valid slots, and the device status word reports MOE_ERR_INVALID_ARG."""
    assert L.moe_device_status() == L.MOE_OK
    for capacity in ("dropless", "ceil_cf_T_over_N"):
        w = replace(SMALL["v3_small"], T=700, N=16, k=4, capacity=capacity, cf=1.5)
        idx = random_routing(w.T, w.N, w.k, "cpu", seed=21).numpy().astype(np.int32)
        idx[3, 1] = w.N + 5                       # out of range
        idx[10, 0] = -1                           # negative
        idx[11, 3] = 1 << 30                      # far out of range
        idx[20, 2] = idx[20, 0]                   # a repeat within the token
        idx[40, :] = w.N                          # every slot invalid: a dropped token
        bad = (idx < 0) | (idx >= w.N)
        bad[20, 2] = True
        clean = np.where(bad, w.N, idx).astype(np.int64)       # invalid slots -> a dummy last expert
        C = O.capacity(oracle_cfg(w), w.T)
        ref = O.permutation(clean, w.N + 1, C)
        c = make_config(w)
        dev = lambda *s_, dtype=torch.int32: torch.full(s_, -7, dtype=dtype, device="cuda")  # noqa: E731
        counts, offsets, ros, tor, nd = dev(w.N), dev(w.N + 1), dev(w.T, w.k), dev(w.T * w.k), dev(2)
        x = torch.randn(w.T, w.d, device="cuda").to(torch.bfloat16)
        xp = torch.zeros(w.T * w.k, w.d, dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(max(L.workspace_size(c), 16), dtype=torch.uint8, device="cuda")
        L.moe_permute(c, x, torch.tensor(idx, device="cuda"), counts, offsets, ros, tor, xp, nd, ws)
        torch.cuda.synchronize()
        assert L.moe_device_status() == L.MOE_ERR_INVALID_ARG      # read and cleared
        assert L.moe_device_status() == L.MOE_OK
        R = int(ref["offsets"][w.N])
        assert np.array_equal(i64(counts), ref["counts"][:w.N])
        assert np.array_equal(i64(offsets), ref["offsets"][:w.N + 1])
        assert np.array_equal(i64(ros), np.where(bad, -1, ref["row_of_slot"]))
        assert np.array_equal(i64(tor)[:R], ref["token_of_row"][:R])
        keep_valid = (~bad) & ref["keep"]
        assert i64(nd).tolist() == [w.T * w.k - R, int((~keep_valid).all(axis=1).sum())]
        assert torch.equal(xp[:R], x[tor[:R].long()])


def test_stats_summed_over_split_batches_equal_whole_batch():
    """Sufficient statistics of two halves of a batch, summed (what the all-reduce
    over data-parallel ranks does) and finalised, equal the statistics of the whole
    batch and the oracle's on all tokens (dropless routing is per token)."""
    w = SMALL["v3_small"]
    inp = make_inputs(w, "cuda")
    whole = MoELayer(w, inp, "cuda", update_bias=False)
    whole.forward(inp["x"])
    half = w.T // 2
    parts = []
    for lo, hi in ((0, half), (half, w.T)):
        wh = replace(w, T=hi - lo)
        lay = MoELayer(wh, dict(inp, x=inp["x"][lo:hi].contiguous()), "cuda", update_bias=False)
        lay.forward(lay.weights["x"])
        L.moe_router_stats_partial(lay.cfg, lay.counts, lay.offsets, lay.p_partial, lay.lse, lay.n_dropped,
                                   lay.stats_part, margin=lay.margin)
        parts.append(lay.stats_part.clone())
    total = parts[0] + parts[1]
    stats = torch.zeros(L.STATS_BYTES, dtype=torch.uint8, device="cuda")
    f_out = torch.empty(w.N, device="cuda")
    p_out = torch.empty(w.N, device="cuda")
    cglob = torch.empty(w.N, dtype=torch.int32, device="cuda")
    L.moe_router_stats_finalize(whole.cfg, total, inp["bias"], w.alpha, w.z_coef, stats, f_out, p_out, cglob)
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    st, st_whole = L.stats_from_tensor(stats), whole.stats_dict()
    assert torch.equal(cglob, whole.counts)
    for key in ("dead", "dropped_slots", "dropped_tokens", "R", "near_ties", "T"):
        assert st[key] == st_whole[key], key
    cfg = oracle_cfg(w)
    r = O.route(f64(inp["x"]), f64(inp["w_gate"]), cfg, bias=f64(inp["bias"]))
    p = O.permutation(i64(whole.topk_idx), w.N, O.capacity(cfg, w.T))
    ost = O.router_stats(p["counts"], p["kept"], r["s"], r["lse"], cfg, w.T, p["dropped_slots"],
                         p["dropped_tokens"], w.alpha, w.z_coef, f64(inp["bias"]))
    for key in ("aux", "aux_raw", "z", "z_loss", "cv", "cv_kept", "bias_norm"):
        assert abs(st[key] - ost[key]) <= TOL_STATS * max(abs(ost[key]), 1e-30) + 1e-12, key
    assert rel_err(f64(f_out), ost["f"]) < TOL_STATS and rel_err(f64(p_out), ost["P"]) < TOL_STATS


@pytest.mark.parametrize("d,f,sizes", [
    (256, 384, [0, 1, 127, 0, 128, 129, 300, 0]),
    # every tile kind: tails of 1..127 rows alone, after one full 128-row tile, after
    # full pairs; partial last n-tiles in both passes (f = 320, d = 384)
    (384, 320, [16, 17, 112, 113, 255, 256, 257, 383, 384, 385, 511, 640, 5, 0, 31]),
])
def test_grouped_ffn_empty_and_tiny_groups(d, f, sizes):
    """Groups with 0, 1, 127, 128, 129 ... rows (every kind of tile: two full 128-row
    sub-tiles, one, one with the group's ragged tail computed transposed, the tail
    alone) and rows_cap beyond the last row."""
    G = len(sizes)
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    R, cap = int(off[-1]), int(off[-1]) + 70
    g = torch.Generator(device="cuda").manual_seed(7)
    xr = torch.randn(cap, d, generator=g, device="cuda").to(torch.bfloat16)
    w1 = (torch.randn(G, f, d, generator=g, device="cuda") / d ** 0.5).to(torch.bfloat16)
    w3 = (torch.randn(G, f, d, generator=g, device="cuda") / d ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn(G, d, f, generator=g, device="cuda") / f ** 0.5).to(torch.bfloat16)
    h = torch.empty(cap, f, dtype=torch.bfloat16, device="cuda")
    y = torch.full((cap, d), 3.0, dtype=torch.bfloat16, device="cuda")
    wk = replace(SMALL["mixtral_small"], d=d, f=f, N=G)
    L.moe_grouped_ffn(make_config(wk), xr, cap, torch.tensor(off, device="cuda"), G, w1, w3, w2, f, h, y)
    torch.cuda.synchronize()
    ref = np.zeros((R, d))
    for e in range(G):
        lo, hi = off[e], off[e + 1]
        if hi > lo:
            ref[lo:hi] = O.swiglu_ffn(f64(xr[lo:hi]), f64(w1[e]), f64(w3[e]), f64(w2[e]))
    assert rel_err(f64(y[:R]), ref) < 2e-2
    for e in range(G):                                 # each group on its own scale
        lo, hi = off[e], off[e + 1]
        if hi > lo:
            assert rel_err(f64(y[lo:hi]), ref[lo:hi]) < 2e-2, (e, sizes[e])
    assert torch.all(y[R:] == 3.0)                     # rows past the last group untouched


@pytest.mark.parametrize("d,f,sizes,Ts,gap", [
    (256, 384, [0, 1, 127, 0, 128, 129, 300, 0], 300, 70),
    (384, 320, [16, 17, 112, 113, 255, 256, 257, 383, 384, 385, 511, 640, 5, 0, 31], 513, 0),
    (256, 256, [0, 0, 0], 129, 5),                       # no routed rows at all
    (256, 256, [40, 200], 16, 1),                        # shared rows: a tail alone
])
def test_grouped_ffn_shared_equals_separate_calls(d, f, sizes, Ts, gap):
    """moe_grouped_ffn_shared (the shared expert as one more group of the same two
    launches) gives bit for bit moe_grouped_ffn on the routed groups plus
    moe_grouped_ffn with G = 1 over x; the shared rows follow the routed rows_cap
    rows, and rows between the last group and rows_cap stay untouched."""
    G = len(sizes)
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    R = int(off[-1])
    cap = R + gap
    g = torch.Generator(device="cuda").manual_seed(5)
    xr = torch.randn(max(cap, 1), d, generator=g, device="cuda").to(torch.bfloat16)
    x = torch.randn(Ts, d, generator=g, device="cuda").to(torch.bfloat16)
    mk = lambda *s, sc: (torch.randn(*s, generator=g, device="cuda") * sc).to(torch.bfloat16)  # noqa: E731
    w1, w3, w2 = mk(G, f, d, sc=d ** -0.5), mk(G, f, d, sc=d ** -0.5), mk(G, d, f, sc=f ** -0.5)
    ws1, ws3, ws2 = mk(f, d, sc=d ** -0.5), mk(f, d, sc=d ** -0.5), mk(d, f, sc=f ** -0.5)
    offs = torch.tensor(off, device="cuda")
    cfg = make_config(replace(SMALL["mixtral_small"], d=d, f=f, N=G, T=Ts))
    h = torch.full((cap + Ts, f), 7.0, dtype=torch.bfloat16, device="cuda")
    y = torch.full((cap + Ts, d), 3.0, dtype=torch.bfloat16, device="cuda")
    L.moe_device_status()
    L.moe_grouped_ffn_shared(cfg, xr, cap, offs, G, w1, w3, w2, f, h, y, x, Ts, ws1, ws3, ws2)
    h0 = torch.empty(max(cap, 1), f, dtype=torch.bfloat16, device="cuda")
    y0 = torch.empty(max(cap, 1), d, dtype=torch.bfloat16, device="cuda")
    if cap > 0:
        L.moe_grouped_ffn(cfg, xr, cap, offs, G, w1, w3, w2, f, h0, y0)
    hs = torch.empty(Ts, f, dtype=torch.bfloat16, device="cuda")
    ys = torch.empty(Ts, d, dtype=torch.bfloat16, device="cuda")
    L.moe_grouped_ffn(cfg, x, Ts, torch.tensor([0, Ts], dtype=torch.int32, device="cuda"), 1, ws1, ws3, ws2, f,
                      hs, ys)
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    assert torch.equal(h[:R], h0[:R]) and torch.equal(y[:R], y0[:R])
    assert torch.equal(h[cap:], hs) and torch.equal(y[cap:], ys)
    assert torch.all(y[R:cap] == 3.0)


@pytest.mark.parametrize("name", ["v3_small"])
def test_layer_fused_shared_expert_equals_separate(name):
    """The layer's output is bit-identical with the shared expert fused into the
    routed launches and with it in launches of its own."""
    w = SMALL[name]
    inp = make_inputs(w, "cuda")
    a = MoELayer(w, inp, "cuda", update_bias=False, fuse_shared=False, overlap_shared=False)
    b = MoELayer(w, inp, "cuda", update_bias=False, fuse_shared=True)
    assert b.fuse_shared and not a.fuse_shared
    ya = a.forward(inp["x"]).clone()
    yb = b.forward(inp["x"])
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    assert torch.equal(ya, yb)
    assert torch.equal(a.ys[:w.T], b.ys[:w.T])


@pytest.mark.parametrize("name", ["v3_small"])
def test_layer_split_shared_expert_equals_fused(name):
    """The shared expert's first pass on a side stream and its second pass inside the
    routed down launch give the fused layer's output bit for bit."""
    w = SMALL[name]
    inp = make_inputs(w, "cuda")
    a = MoELayer(w, inp, "cuda", update_bias=False, fuse_shared=True, split_shared=False)
    b = MoELayer(w, inp, "cuda", update_bias=False, fuse_shared=True, split_shared=True)
    assert b.split_shared and not a.split_shared
    ya = a.forward(inp["x"]).clone()
    for _ in range(2):
        yb = b.forward(inp["x"]).clone()
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    assert torch.equal(ya, yb)
    assert torch.equal(a.ys[:w.T], b.ys[:w.T])


@pytest.mark.parametrize("d,f,sizes,T", [
    (256, 384, [0, 1, 127, 0, 128, 129, 300, 0], 613),
    (384, 256, [16, 17, 255, 256, 257, 5], 200),
])
def test_grouped_ffn_passes_equal_fused_shared(d, f, sizes, T):
    """moe_grouped_ffn_gate_up on the routed rows and on x (the shared expert), then
    moe_grouped_ffn_down with the shared weights, equal moe_grouped_ffn_shared bit for bit."""
    G = len(sizes)
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    R, cap = int(off[-1]), int(off[-1]) + 40
    g = torch.Generator(device="cuda").manual_seed(31)
    x = torch.randn(T, d, generator=g, device="cuda").to(torch.bfloat16)
    xr = torch.randn(cap, d, generator=g, device="cuda").to(torch.bfloat16)
    w1 = (torch.randn(G, f, d, generator=g, device="cuda") / d ** 0.5).to(torch.bfloat16)
    w3 = (torch.randn(G, f, d, generator=g, device="cuda") / d ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn(G, d, f, generator=g, device="cuda") / f ** 0.5).to(torch.bfloat16)
    ws1 = (torch.randn(f, d, generator=g, device="cuda") / d ** 0.5).to(torch.bfloat16)
    ws3 = (torch.randn(f, d, generator=g, device="cuda") / d ** 0.5).to(torch.bfloat16)
    ws2 = (torch.randn(d, f, generator=g, device="cuda") / f ** 0.5).to(torch.bfloat16)
    offs = torch.tensor(off, device="cuda")
    cfg = make_config(replace(SMALL["mixtral_small"], d=d, f=f, N=G, T=T))
    h0, h1 = (torch.empty(cap + T, f, dtype=torch.bfloat16, device="cuda") for _ in range(2))
    y0, y1 = (torch.full((cap + T, d), 3.0, dtype=torch.bfloat16, device="cuda") for _ in range(2))
    L.moe_device_status()
    L.moe_grouped_ffn_shared(cfg, xr, cap, offs, G, w1, w3, w2, f, h0, y0, x, T, ws1, ws3, ws2)
    L.moe_grouped_ffn_gate_up(cfg, x, T, torch.tensor([0, T], dtype=torch.int32, device="cuda"), 1, ws1, ws3, f,
                              h1[cap:])
    L.moe_grouped_ffn_gate_up(cfg, xr, cap, offs, G, w1, w3, f, h1)
    L.moe_grouped_ffn_down(cfg, h1, cap, offs, G, w2, f, y1, T, ws2)
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    assert torch.equal(h1[:R], h0[:R]) and torch.equal(h1[cap:], h0[cap:])
    assert torch.equal(y1, y0)


@pytest.mark.parametrize("d,f,sizes", [
    (256, 384, [0, 1, 127, 0, 128, 129, 300, 0]),
    (384, 320, [16, 17, 112, 113, 255, 256, 257, 383, 384, 385, 511, 640, 5, 0, 31]),
])
def test_grouped_ffn_gather_equals_grouped_ffn_on_gathered_rows(d, f, sizes):
    """moe_grouped_ffn_gather (rows fetched from x by index inside the first GEMM) gives
    bit for bit what moe_grouped_ffn gives on the gathered rows x[token_of_row], over
    every tile kind; rows past the last group stay untouched."""
    G = len(sizes)
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    R, cap = int(off[-1]), int(off[-1]) + 70
    T = 613
    g = torch.Generator(device="cuda").manual_seed(11)
    x = torch.randn(T, d, generator=g, device="cuda").to(torch.bfloat16)
    # repeats and arbitrary order, as a permutation's row map has; entries >= R are
    # never read, so they hold an out-of-range id
    tor = torch.randint(0, T, (cap,), generator=g, device="cuda", dtype=torch.int32)
    tor[R:] = T + 5
    w1 = (torch.randn(G, f, d, generator=g, device="cuda") / d ** 0.5).to(torch.bfloat16)
    w3 = (torch.randn(G, f, d, generator=g, device="cuda") / d ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn(G, d, f, generator=g, device="cuda") / f ** 0.5).to(torch.bfloat16)
    offs = torch.tensor(off, device="cuda")
    cfg = make_config(replace(SMALL["mixtral_small"], d=d, f=f, N=G, T=T))
    xr = torch.zeros(cap, d, dtype=torch.bfloat16, device="cuda")
    xr[:R] = x[tor[:R].long()]
    h0, h1 = (torch.empty(cap, f, dtype=torch.bfloat16, device="cuda") for _ in range(2))
    y0, y1 = (torch.full((cap, d), 3.0, dtype=torch.bfloat16, device="cuda") for _ in range(2))
    L.moe_device_status()
    L.moe_grouped_ffn(cfg, xr, cap, offs, G, w1, w3, w2, f, h0, y0)
    L.moe_grouped_ffn_gather(cfg, x, T, tor, cap, offs, G, w1, w3, w2, f, h1, y1)
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    assert torch.equal(h1[:R], h0[:R])
    assert torch.equal(y1, y0)
    assert torch.all(y0[R:] == 3.0)                # no output row past the last group is written


@pytest.mark.parametrize("d,f,sizes,T", [
    (256, 384, [0, 1, 127, 0, 128, 129, 300, 0], 613),
    (384, 256, [16, 17, 255, 256, 257, 5], 200),
])
def test_grouped_ffn_gather_with_shared_expert(d, f, sizes, T):
    """moe_grouped_ffn_gather with the shared weights equals moe_grouped_ffn_shared on
    the gathered rows bit for bit: routed rows and the shared expert's T rows after
    them, every tile kind of both."""
    G = len(sizes)
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    R, cap = int(off[-1]), int(off[-1]) + 40
    g = torch.Generator(device="cuda").manual_seed(21)
    x = torch.randn(T, d, generator=g, device="cuda").to(torch.bfloat16)
    tor = torch.randint(0, T, (cap,), generator=g, device="cuda", dtype=torch.int32)
    w1 = (torch.randn(G, f, d, generator=g, device="cuda") / d ** 0.5).to(torch.bfloat16)
    w3 = (torch.randn(G, f, d, generator=g, device="cuda") / d ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn(G, d, f, generator=g, device="cuda") / f ** 0.5).to(torch.bfloat16)
    ws1 = (torch.randn(f, d, generator=g, device="cuda") / d ** 0.5).to(torch.bfloat16)
    ws3 = (torch.randn(f, d, generator=g, device="cuda") / d ** 0.5).to(torch.bfloat16)
    ws2 = (torch.randn(d, f, generator=g, device="cuda") / f ** 0.5).to(torch.bfloat16)
    offs = torch.tensor(off, device="cuda")
    cfg = make_config(replace(SMALL["mixtral_small"], d=d, f=f, N=G, T=T))
    xr = torch.zeros(cap, d, dtype=torch.bfloat16, device="cuda")
    xr[:R] = x[tor[:R].long()]
    h0, h1 = (torch.empty(cap + T, f, dtype=torch.bfloat16, device="cuda") for _ in range(2))
    y0, y1 = (torch.full((cap + T, d), 3.0, dtype=torch.bfloat16, device="cuda") for _ in range(2))
    L.moe_device_status()
    L.moe_grouped_ffn_shared(cfg, xr, cap, offs, G, w1, w3, w2, f, h0, y0, x, T, ws1, ws3, ws2)
    L.moe_grouped_ffn_gather(cfg, x, T, tor, cap, offs, G, w1, w3, w2, f, h1, y1, ws1=ws1, ws3=ws3, ws2=ws2)
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    assert torch.equal(h1[:R], h0[:R]) and torch.equal(h1[cap:], h0[cap:])
    assert torch.equal(y1, y0)


def test_grouped_ffn_gather_flags_out_of_range_token_ids():
    """A token id outside [0, T) in a read row is replaced by token 0 and recorded
    as MOE_ERR_INVALID_ARG; the call itself completes."""
    d, f, sizes = 256, 256, [130, 5]
    G = len(sizes)
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    R, T = int(off[-1]), 50
    g = torch.Generator(device="cuda").manual_seed(3)
    x = torch.randn(T, d, generator=g, device="cuda").to(torch.bfloat16)
    tor = torch.randint(0, T, (R,), generator=g, device="cuda", dtype=torch.int32)
    tor[7], tor[R - 1] = T, -1
    w1 = (torch.randn(G, f, d, generator=g, device="cuda") / d ** 0.5).to(torch.bfloat16)
    w3 = (torch.randn(G, f, d, generator=g, device="cuda") / d ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn(G, d, f, generator=g, device="cuda") / f ** 0.5).to(torch.bfloat16)
    cfg = make_config(replace(SMALL["mixtral_small"], d=d, f=f, N=G, T=T))
    h = torch.empty(R, f, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(R, d, dtype=torch.bfloat16, device="cuda")
    L.moe_device_status()
    L.moe_grouped_ffn_gather(cfg, x, T, tor, R, torch.tensor(off, device="cuda"), G, w1, w3, w2, f, h, y)
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_ERR_INVALID_ARG
    fixed = tor.clone()
    fixed[7], fixed[R - 1] = 0, 0
    y_ok = torch.empty_like(y)
    L.moe_grouped_ffn_gather(cfg, x, T, fixed, R, torch.tensor(off, device="cuda"), G, w1, w3, w2, f, h, y_ok)
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    assert torch.equal(y, y_ok)


@pytest.mark.parametrize("name", ["mixtral_small", "v3_small", "switch_small"])
def test_layer_gathering_ffn_equals_permuted_copy(name):
    """The layer's output is bit-identical whether the grouped FFN reads the permuted
    copy of x or gathers its rows from x."""
    w = SMALL[name]
    inp = make_inputs(w, "cuda")
    a = MoELayer(w, inp, "cuda", update_bias=False, gather_rows=False)
    b = MoELayer(w, inp, "cuda", update_bias=False, gather_rows=True)
    assert a.x_perm is not None and b.x_perm is None
    ya = a.forward(inp["x"]).clone()
    yb = b.forward(inp["x"])
    torch.cuda.synchronize()
    assert torch.equal(ya, yb)
    assert torch.equal(a.y_perm[:int(a.offsets[-1])], b.y_perm[:int(b.offsets[-1])])


# ----------------------------------------------------------------------------- full size
FULL = ["mixtral_8x7b", "deepseekmoe_16b", "deepseek_v3", "switch_skewed"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_workload(name):
    w = WORKLOADS[name]
    lay, inp, _ = _run(w)
    rng = np.random.default_rng(0)
    sample = np.sort(rng.choice(w.T, size=min(w.T, 512), replace=False))
    n_tie, r = _check_route(w, lay, inp, sample)
    print(f"{name}: near-ties {n_tie}/{len(sample)} sampled tokens")
    p = _check_permute(w, lay, inp)
    # expert rows: 8 experts (the most and least loaded included), up to 48 rows each
    off = i64(lay.offsets)
    loads = np.diff(off)
    pick = sorted(set([int(np.argmax(loads)), int(np.argmin(np.where(loads > 0, loads, 1 << 30)))] +
                      rng.choice(w.N, size=min(w.N, 6), replace=False).tolist()))
    rows = {}
    for e in pick:
        n = int(loads[e])
        if n:
            sel = np.unique(np.concatenate([[0, n - 1], rng.choice(n, size=min(n, 46), replace=False)]))
            rows[e] = torch.tensor(off[e] + sel, device="cuda")
    _check_ffn_rows(w, lay, inp, rows)
    # combine + whole layer on sampled tokens, oracle fed the GPU's expert choice
    tok = sample[:24]
    cfg = oracle_cfg(w)
    s = O.affinity(O.router_logits(f64(inp["x"][torch.tensor(tok, device="cuda")]), f64(inp["w_gate"]),
                                   f64(inp["logit_offset"])), cfg.score_fn)
    wts = np.zeros((w.T, w.k))
    wts[tok] = O.gate_weights(s, i64(lay.topk_idx)[tok], cfg.renorm)
    out = O.layer_forward(f64(inp["x"]), None, cfg, expert_weights_fn(inp), shared_weights(inp),
                          tokens=tok, routing={"idx": i64(lay.topk_idx), "w": wts})
    assert rel_err(f64(lay.y[torch.tensor(tok, device="cuda")]), out["y"]) < tol_for(w)
    # statistics on every token: the oracle routes all T tokens in fp64 (its own
    # affinities and lse), counts and drops from the GPU's expert choice (cross-fed)
    rall = O.route(f64(inp["x"]), f64(inp["w_gate"]), cfg, bias=f64(inp["bias"]),
                   logit_offset=f64(inp["logit_offset"]))
    ost = O.router_stats(p["counts"], p["kept"], rall["s"], rall["lse"], cfg, w.T, p["dropped_slots"],
                         p["dropped_tokens"], w.alpha, w.z_coef, f64(inp["bias"]))
    st = lay.stats_dict()
    for key in ("aux", "aux_raw", "z", "z_loss", "cv", "cv_kept", "bias_norm"):
        assert abs(st[key] - ost[key]) <= TOL_STATS * max(abs(ost[key]), 1e-30) + 1e-12, key
    for key in ("dead", "dropped_slots", "dropped_tokens"):
        assert st[key] == ost[key], key
    assert st["R"] == p["R"] and st["T"] == w.T
    assert rel_err(f64(lay.f_out), ost["f"]) < TOL_STATS
    assert rel_err(f64(lay.p_out), ost["P"]) < TOL_STATS
    n_oracle = _check_near_ties(st, lay, rall["margin"])
    print(f"{name}: near-ties {st['near_ties']} (oracle {n_oracle}) of {w.T} tokens")


def test_forward_host_pipeline_matches_forward():
    """Pinned host in/out with overlapped copies gives each step's own result."""
    w = replace(SMALL["v3_small"], T=640)
    inp = make_inputs(w, "cuda")
    lay = MoELayer(w, inp, "cuda", update_bias=False)
    g = torch.Generator(device="cuda").manual_seed(5)
    xs = [torch.randn(w.T, w.d, generator=g, device="cuda").to(torch.bfloat16) for _ in range(3)]
    want = []
    for x in xs:
        want.append(lay.forward(x).clone())
    xh = [x.cpu().pin_memory() for x in xs]
    yh = [torch.empty(w.T, w.d, dtype=torch.bfloat16).pin_memory() for _ in xs]
    lay.forward_host(xh, yh)
    torch.cuda.synchronize()
    for a, b in zip(want, yh):
        assert torch.equal(a.cpu(), b)


def test_cuda_graph_replay_matches_eager():
    """A captured forward replays the same launches: outputs and the bias after the
    same number of steps are bit-identical to eager execution."""
    w = replace(SMALL["v3_small"], T=513)
    inp_a = make_inputs(w, "cuda")
    inp_b = make_inputs(w, "cuda")
    eager = MoELayer(w, inp_a, "cuda", update_bias=True)
    graph = MoELayer(w, inp_b, "cuda", update_bias=True)
    graph.capture(inp_b["x"])                  # one eager forward + the capture
    eager.forward(inp_a["x"])
    for _ in range(3):
        eager.forward(inp_a["x"])
        graph.replay()
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    assert torch.equal(eager.y, graph.y)
    assert torch.equal(inp_a["bias"], inp_b["bias"])
    assert torch.equal(eager.stats, graph.stats)


def test_route_with_prepared_split_equals_route_with_weight():
    """moe_route on the split written once by moe_route_prepare (w_gate = NULL) gives
    the same bytes as moe_route splitting w_gate itself."""
    w = SMALL["v3_small"]
    inp = make_inputs(w, "cuda")
    c = make_config(w)
    T, N, k = w.T, w.N, w.k
    nblk = L.route_partials(c)
    outs = []
    for prepared in (False, True):
        z = lambda *s, dtype=torch.float32: torch.full(s, -3, dtype=dtype, device="cuda")  # noqa: E731
        o = [z(T, k, dtype=torch.int32), z(T, k), z(T), z(nblk, N), z(T)]
        ws = torch.zeros(max(L.workspace_size(c), 16), dtype=torch.uint8, device="cuda")
        if prepared:
            L.moe_route_prepare(c, inp["w_gate"], ws)
        L.moe_route(c, inp["x"], None if prepared else inp["w_gate"], None, inp["bias"], *o, ws)
        outs.append(o)
    torch.cuda.synchronize()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_permute_row_sizes_in_any_order():
    """Calls whose rows need different amounts of dynamic shared memory, larger after
    smaller: a kernel's shared-memory limit is only ever raised, never lowered."""
    for d in (512, 264, 512, 1024, 264):
        w = replace(SMALL["mixtral_small"], d=d, T=300)
        inp = make_inputs(w, "cuda", experts=False)
        c = make_config(w)
        T, N, k = w.T, w.N, w.k
        idx = torch.stack([torch.arange(T, device="cuda") % N, (torch.arange(T, device="cuda") + 3) % N],
                          1).to(torch.int32).contiguous()
        z = lambda *s: torch.zeros(*s, dtype=torch.int32, device="cuda")  # noqa: E731
        counts, offsets, ros, tor, nd = z(N), z(N + 1), z(T, k), z(T * k), z(2)
        xp = torch.zeros(T * k, d, dtype=torch.bfloat16, device="cuda")
        ws = torch.zeros(max(L.workspace_size(c), 16), dtype=torch.uint8, device="cuda")
        L.moe_permute(c, inp["x"], idx, counts, offsets, ros, tor, xp, nd, ws)
        torch.cuda.synchronize()
        R = int(offsets[-1])
        assert R == T * k
        assert torch.equal(xp[:R], inp["x"][tor[:R].long()])
