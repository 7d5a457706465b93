"""GPU-vs-oracle parity of the MXFP8 expert path, through the C ABI.

Quantisation (E4M3 codes and E8M0 scale bytes) is compared bit for bit: the
scale exponent is an integer decision both sides take from the same fp32 amax,
and x / 2^e is exact.  h is re-quantised from the GPU's fp32 GEMM and the
oracle's fp64 one, so it is checked within the E4M3 rounding bound; y against the
oracle's down projection of the GPU's own h and against the oracle's MXFP8 expert
end to end.
"""
from __future__ import annotations

from dataclasses import replace

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_21_b200 import _lib as L
from sparse_mixture_experts_21_b200.layer import MoELayer, make_config
from sparse_mixture_experts_21_b200.synth import WORKLOADS, make_inputs
from tests.parity_util import (NEAR_TIE, expert_weights_fn, f64, i64, mx_scales_rowmajor, oracle_cfg, rel_err,
                               shared_weights)
from tests.test_gpu_fp8 import decode_e4m3

pytestmark = pytest.mark.gpu

TOL_MX = 2e-2           # y vs the oracle's MXFP8 expert
TOL_MX_SAME_H = 5e-3    # y vs the oracle's down projection of the GPU's own h codes
# The block-scaled MMA accumulates the whole K range inside the tensor core (no fp32
# register accumulation between K blocks), which keeps fewer bits than fp32: h may
# differ from the fp64 GEMM by up to 2^-8 of its 32-block's largest magnitude on top
# of the E4M3 rounding, and a few more codes may round the other way.
ACC_MX = 2.0 ** -8


def gpu_mx(x: torch.Tensor):
    R, C = x.shape
    q = torch.empty(R, C, dtype=torch.uint8, device="cuda")
    sf = L.mx_scales(R, C, "cuda")
    L.moe_quantize_mxfp8(x, q, sf)
    return q, sf


def exps(sf: torch.Tensor, rows: int, cols: int, offsets=None) -> np.ndarray:
    """GPU scale bytes (tile atoms) -> exponents [rows, cols / 32]."""
    return mx_scales_rowmajor(sf, rows, cols, offsets).astype(np.int64) - 127


def deq_mx(q: torch.Tensor, sf: torch.Tensor, offsets=None) -> np.ndarray:
    R, C = q.shape
    return O.dequantize_mxfp8(decode_e4m3(q.cpu().numpy()), exps(sf, R, C, offsets))


def test_mx_quantize_bit_exact():
    g = torch.Generator(device="cuda").manual_seed(7)
    R, C = 300, 640
    x = torch.randn(R, C, generator=g, device="cuda") * torch.exp2(torch.randint(-12, 12, (R, 1), generator=g,
                                                                                device="cuda").float())
    x[3, :32] = 0.0                                     # an all-zero block
    x[4, 64:96] = 448.0                                 # amax exactly 2^8 * 1.75
    x[5, 96:128] = 2.0                                  # an exact power of two
    x[6, 7] = 500.0                                     # saturates
    xb = x.to(torch.bfloat16)
    q, sf = gpu_mx(xb)
    torch.cuda.synchronize()
    q_ref, e_ref = O.quantize_mxfp8(f64(xb))
    assert np.array_equal(exps(sf, R, C), e_ref)
    assert np.array_equal(decode_e4m3(q.cpu().numpy()), q_ref)


def _mx_layer_case():
    return replace(WORKLOADS["deepseekmoe_16b"], name="dsmoe_mx_small", T=777, d=384, N=16, k=6,
                   f=256, n_shared=1, f_shared=384, mxfp8=True)


def test_permute_mxfp8_rows_bit_exact():
    w = _mx_layer_case()
    inp = make_inputs(w, "cuda")
    lay = MoELayer(w, inp, "cuda", update_bias=False)
    c = lay.cfg
    L.moe_route(c, inp["x"], inp["w_gate"], None, inp.get("bias"), lay.topk_idx, lay.topk_w, lay.lse,
                lay.p_partial, lay.margin, lay.ws)
    L.moe_permute(c, None, lay.topk_idx, lay.counts, lay.offsets, lay.row_of_slot, lay.token_of_row, None,
                  lay.n_dropped, lay.ws)
    L.moe_permute_mxfp8(c, inp["x"], lay.topk_idx, lay.row_of_slot, lay.offsets, lay.xq_perm, lay.xs_perm,
                        lay.xq, lay.xs)
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    q_ref, e_ref = O.quantize_mxfp8(f64(inp["x"]))
    R = int(lay.offsets[-1].item())
    tor = i64(lay.token_of_row)[:R]
    off = i64(lay.offsets)
    assert np.array_equal(decode_e4m3(lay.xq_perm[:R].cpu().numpy()), q_ref[tor])
    assert np.array_equal(exps(lay.xs_perm, R, w.d, off), e_ref[tor])
    assert np.array_equal(decode_e4m3(lay.xq[:w.T].cpu().numpy()), q_ref)
    assert np.array_equal(exps(lay.xs, w.T, w.d), e_ref)


@pytest.mark.parametrize("d,f,sizes", [
    (384, 384, [0, 1, 130, 257, 77]),        # empty and 1-row groups, ragged tails, 2 N tiles of y
    (256, 512, [128, 0, 0, 300]),
    (7168, 2048, [5, 0, 190]),                # the DeepSeek-V3 expert shape
])
def test_grouped_ffn_mxfp8(d, f, sizes):
    G = len(sizes)
    R = sum(sizes)
    rows_cap = R + 40
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    gen = torch.Generator(device="cuda").manual_seed(d + 3 * f + G)
    rnd = lambda *s, std=1.0: (torch.randn(*s, generator=gen, device="cuda") * std).to(torch.bfloat16)  # noqa
    x = rnd(rows_cap, d)
    w1, w3 = rnd(G, f, d, std=d ** -0.5), rnd(G, f, d, std=d ** -0.5)
    w2 = rnd(G, d, f, std=f ** -0.5)
    # x in the grouped tile-atom order: quantise each group's rows on their own
    xq = torch.empty(rows_cap, d, dtype=torch.uint8, device="cuda")
    xsf = L.mx_scales(rows_cap, d, "cuda", G)
    nkb = d // 128
    tile = 0
    for g in range(G):
        n = int(off[g + 1] - off[g])
        if n == 0:
            continue
        qg, sg = gpu_mx(x[off[g]:off[g + 1]])
        xq[off[g]:off[g + 1]] = qg
        nt = (n + 127) // 128
        xsf[tile * nkb * 512:(tile + nt) * nkb * 512] = sg[:nt * nkb * 512]
        tile += nt
    (w1q, w1sf), (w3q, w3sf), (w2q, w2sf) = (gpu_mx(t.reshape(-1, t.shape[-1])) for t in (w1, w3, w2))
    hq = torch.zeros(rows_cap, f, dtype=torch.uint8, device="cuda")
    hsf = L.mx_scales(rows_cap, f, "cuda", G).zero_()
    y = torch.full((rows_cap, d), 7.0, dtype=torch.bfloat16, device="cuda")
    cfg = make_config(replace(WORKLOADS["deepseek_v3"], d=d, T=R))
    L.moe_grouped_ffn_mxfp8(cfg, xq, xsf, rows_cap, torch.tensor(off, device="cuda"), G, w1q, w1sf, w3q, w3sf,
                            w2q, w2sf, f, hq, hsf, y)
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    assert torch.all(y[R:] == 7.0)
    x64 = f64(x)
    h_gpu = deq_mx(hq[:R], hsf, off)
    e_h = exps(hsf, R, f, off)
    y_gpu = f64(y)
    checked = 0
    for g in range(G):
        lo, hi = off[g], off[g + 1]
        if hi == lo:
            continue
        xd = O.dequantize_mxfp8(*O.quantize_mxfp8(x64[lo:hi]))
        wd = [O.dequantize_mxfp8(*O.quantize_mxfp8(f64(t[g]))) for t in (w1, w3, w2)]
        h_ref = O.silu(xd @ wd[0].T) * (xd @ wd[1].T)
        amax = np.repeat(np.abs(h_ref).reshape(hi - lo, -1, 32).max(axis=2), 32, axis=1)
        err = np.abs(h_gpu[lo:hi] - h_ref)
        # the oracle's rounding of h_ref under the GPU's own block exponents (saturation
        # included: a block's largest element may exceed 448 * 2^e and clamp)
        q_same = np.repeat(2.0 ** e_h[lo:hi], 32, axis=1) * O.round_e4m3(
            h_ref / np.repeat(2.0 ** e_h[lo:hi], 32, axis=1))
        one_ulp = 2.0 ** -3 * np.abs(q_same) + np.repeat(2.0 ** (e_h[lo:hi] - 9), 32, axis=1)
        err = np.abs(h_gpu[lo:hi] - h_ref)
        excess = float(np.max((err - np.abs(q_same - h_ref)) / amax))
        assert np.all(err <= np.abs(q_same - h_ref) + one_ulp + ACC_MX * amax), excess
        codes_ref, e_ref = O.quantize_mxfp8(h_ref)
        same_e = np.mean(e_h[lo:hi] == e_ref)
        same = np.mean(h_gpu[lo:hi] == q_same)
        print(f"group {g}: rows {hi - lo}, error beyond the oracle's rounding {excess:.2e} of block amax, "
              f"exponents equal {same_e:.4f}, values equal {same:.4f}")
        assert same_e >= 0.99 and same >= 0.97, (same_e, same)
        assert rel_err(y_gpu[lo:hi], h_gpu[lo:hi] @ wd[2].T) < TOL_MX_SAME_H
        y_ref = O.swiglu_ffn_mxfp8(x64[lo:hi], f64(w1[g]), f64(w3[g]), f64(w2[g]))
        assert rel_err(y_gpu[lo:hi], y_ref) < TOL_MX
        checked += hi - lo
    assert checked == R


def test_mxfp8_layer_forward():
    w = _mx_layer_case()
    inp = make_inputs(w, "cuda")
    lay = MoELayer(w, inp, "cuda", update_bias=False)
    lay.forward(inp["x"])
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    cfg = oracle_cfg(w)
    r = O.route(f64(inp["x"]), f64(inp["w_gate"]), cfg, f64(inp.get("bias")))
    clear = r["margin"] >= NEAR_TIE
    assert np.array_equal(i64(lay.topk_idx)[clear], r["idx"][clear])
    out = O.layer_forward(f64(inp["x"]), None, cfg, expert_weights_fn(inp), shared_weights(inp),
                          routing={"idx": i64(lay.topk_idx), "w": f64(lay.topk_w)},
                          expert_ffn=O.swiglu_ffn_mxfp8)
    assert rel_err(f64(lay.y[:w.T]), out["y"]) < TOL_MX


def test_mxfp8_deepseek_v3_sampled_tokens():
    w = WORKLOADS["deepseek_v3_mxfp8"]
    inp = make_inputs(w, "cuda")
    lay = MoELayer(w, inp, "cuda", update_bias=False)
    lay.forward(inp["x"])
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    toks = np.random.default_rng(2).choice(w.T, size=4, replace=False)
    get = expert_weights_fn(inp)
    idx, wts = i64(lay.topk_idx), f64(lay.topk_w)
    x64 = f64(inp["x"])
    y_gpu = f64(lay.y[torch.tensor(toks, device="cuda")])
    y_ref = O.swiglu_ffn_mxfp8(x64[toks], *shared_weights(inp))
    by_expert = {}
    for i, t in enumerate(toks):
        for j in range(w.k):
            by_expert.setdefault(int(idx[t, j]), []).append((i, j))
    for e, uses in by_expert.items():
        ye = O.swiglu_ffn_mxfp8(x64[toks[[i for i, _ in uses]]], *get(e))
        for r_i, (i, j) in enumerate(uses):
            y_ref[i] += wts[toks[i], j] * ye[r_i]
    for i, t in enumerate(toks):
        assert rel_err(y_gpu[i], y_ref[i]) < TOL_MX, (t, rel_err(y_gpu[i], y_ref[i]))
