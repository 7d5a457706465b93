"""GPU-vs-oracle parity of the FP8 expert path, through the C ABI.

Block quantisation (codes and scales) is compared bit for bit: both sides divide
in fp32 and round to E4M3 with ties to even.  The hidden activations h are
re-quantised from an fp32 GEMM on the GPU and an fp64 one in the oracle, so their
codes may differ where h / s sits on a rounding boundary: h is checked against the
oracle within the E4M3 rounding bound, and y against the oracle's down projection
of the GPU's own h codes (tight) and against the oracle's FP8 expert end to end.
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
from tests.parity_util import NEAR_TIE, expert_weights_fn, f64, i64, oracle_cfg, rel_err, shared_weights

pytestmark = pytest.mark.gpu

TOL_FP8 = 2e-2          # y vs the oracle's FP8 expert (same quantisation reading)
TOL_FP8_SAME_H = 5e-3   # y vs the oracle's down projection of the GPU's own h codes


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    """E4M3 bit pattern -> value: sign bit 7, exponent bits 6..3 (bias 7), mantissa
    bits 2..0; exponent 0 is subnormal (m 2^-9); 0x7F / 0xFF are NaN."""
    c = np.asarray(codes, np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * 2.0 ** (e - 7))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return sign * val


def gpu_quant(x: torch.Tensor, block_rows: int):
    R, C = x.shape
    q = torch.empty(R, C, dtype=torch.uint8, device="cuda")
    s = torch.empty((R + block_rows - 1) // block_rows, C // 128, dtype=torch.float32, device="cuda")
    L.moe_quantize_fp8(x, block_rows, q, s)
    return q, s


def deq(q: torch.Tensor, s: torch.Tensor, block_rows: int) -> np.ndarray:
    return O.dequantize_fp8_blocks(decode_e4m3(q.cpu().numpy()), s.cpu().numpy(), block_rows)


@pytest.mark.parametrize("block_rows", [1, 128])
def test_quantize_bit_exact(block_rows):
    g = torch.Generator(device="cuda").manual_seed(5)
    R, C = 300, 640
    x = torch.randn(R, C, generator=g, device="cuda")
    x[7, :128] = 0.0                                    # an all-zero 1 x 128 block
    x[:128, 256:384] = 0.0                              # an all-zero 128 x 128 block
    x[9, 130] = 3.0e4                                   # a wide-range block
    x[200:210] *= 1e-3                                  # subnormal codes in 1 x 128 blocks
    xb = x.to(torch.bfloat16)
    q, s = gpu_quant(xb, block_rows)
    torch.cuda.synchronize()
    q_ref, s_ref = O.quantize_fp8_blocks(f64(xb), block_rows)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(decode_e4m3(q.cpu().numpy()), q_ref)
    assert not np.any((q.cpu().numpy() & 0x7F) == 0x7F)  # never NaN


def _fp8_layer_case():
    return replace(WORKLOADS["deepseekmoe_16b"], name="dsmoe_fp8_small", T=777, d=384, N=16, k=6,
                   f=256, n_shared=1, f_shared=384, fp8=True)


def test_permute_fp8_rows_bit_exact():
    w = _fp8_layer_case()
    inp = make_inputs(w, "cuda")
    lay = MoELayer(w, inp, "cuda", update_bias=False)
    c = lay.cfg
    L.moe_route(c, inp["x"], inp["w_gate"], None, inp.get("bias"), lay.topk_idx, lay.topk_w, lay.lse,
                lay.p_partial, lay.margin, lay.ws)
    L.moe_permute(c, None, lay.topk_idx, lay.counts, lay.offsets, lay.row_of_slot, lay.token_of_row, None,
                  lay.n_dropped, lay.ws)
    L.moe_permute_fp8(c, inp["x"], lay.row_of_slot, lay.xq_perm, lay.xs_perm, lay.xq, lay.xs)
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    q_ref, s_ref = O.quantize_fp8_blocks(f64(inp["x"]), 1)
    R = int(lay.offsets[-1].item())
    tor = i64(lay.token_of_row)[:R]
    assert R == w.T * w.k
    assert np.array_equal(decode_e4m3(lay.xq_perm[:R].cpu().numpy()), q_ref[tor])
    assert np.array_equal(lay.xs_perm[:R].cpu().numpy(), s_ref[tor])
    assert np.array_equal(decode_e4m3(lay.xq[:w.T].cpu().numpy()), q_ref)
    assert np.array_equal(lay.xs[:w.T].cpu().numpy(), s_ref)


@pytest.mark.parametrize("d,f,sizes", [
    (384, 384, [0, 1, 130, 257, 77]),        # empty and 1-row groups, ragged tails, 2 N tiles of y
    (256, 512, [128, 0, 0, 300]),
    (7168, 2048, [5, 0, 190]),                # the DeepSeek-V3 expert shape, 56 / 16 K blocks
])
def test_grouped_ffn_fp8(d, f, sizes):
    G = len(sizes)
    R = sum(sizes)
    rows_cap = R + 40
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    gen = torch.Generator(device="cuda").manual_seed(d + f + G)
    rnd = lambda *s, std=1.0: (torch.randn(*s, generator=gen, device="cuda") * std).to(torch.bfloat16)  # noqa
    x = rnd(rows_cap, d)
    w1, w3 = rnd(G, f, d, std=d ** -0.5), rnd(G, f, d, std=d ** -0.5)
    w2 = rnd(G, d, f, std=f ** -0.5)
    xq, xs = gpu_quant(x, 1)
    (w1q, w1s), (w3q, w3s), (w2q, w2s) = (gpu_quant(t.reshape(-1, t.shape[-1]), 128) for t in (w1, w3, w2))
    hq = torch.zeros(rows_cap, f, dtype=torch.uint8, device="cuda")
    hs = torch.zeros(rows_cap, f // 128, device="cuda")
    y = torch.full((rows_cap, d), 7.0, dtype=torch.bfloat16, device="cuda")
    cfg = make_config(replace(WORKLOADS["deepseek_v3"], d=d, T=R))
    L.moe_grouped_ffn_fp8(cfg, xq, xs, rows_cap, torch.tensor(off, device="cuda"), G, w1q, w1s, w3q, w3s,
                          w2q, w2s, f, hq, hs, y)
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    assert torch.all(y[R:] == 7.0)                     # rows past the last group untouched
    x64 = f64(x)
    h_gpu = deq(hq, hs, 1)
    y_gpu = f64(y)
    checked = 0
    for g in range(G):
        lo, hi = off[g], off[g + 1]
        if hi == lo:
            continue
        # oracle on the oracle's own quantisation of the same bf16 inputs
        xd = O.dequantize_fp8_blocks(*O.quantize_fp8_blocks(x64[lo:hi], 1), 1)
        wd = [O.dequantize_fp8_blocks(*O.quantize_fp8_blocks(f64(t[g]), 128), 128) for t in (w1, w3, w2)]
        h_ref = O.silu(xd @ wd[0].T) * (xd @ wd[1].T)
        # h within the E4M3 bound: half an ulp (2^-4 relative for normals, 2^-10 s
        # for subnormals) plus the fp32 accumulation and the scale's own rounding
        s_blk = np.repeat(hs[lo:hi].cpu().numpy().astype(np.float64), 128, axis=1)
        amax = np.repeat(np.abs(h_ref).reshape(hi - lo, -1, 128).max(axis=2), 128, axis=1)
        err = np.abs(h_gpu[lo:hi] - h_ref)
        assert np.all(err <= 2.0 ** -4 * np.abs(h_ref) + 2.0 ** -10 * s_blk + 1e-4 * amax)
        codes_ref = O.quantize_fp8_blocks(h_ref, 1)[0]
        same = np.mean(decode_e4m3(hq[lo:hi].cpu().numpy()) == codes_ref)
        assert same >= 0.995, same
        # y: the oracle's down projection of the GPU's own h codes, then end to end
        assert rel_err(y_gpu[lo:hi], h_gpu[lo:hi] @ wd[2].T) < TOL_FP8_SAME_H
        y_ref = O.swiglu_ffn_fp8(x64[lo:hi], f64(w1[g]), f64(w3[g]), f64(w2[g]))
        assert rel_err(y_gpu[lo:hi], y_ref) < TOL_FP8
        checked += hi - lo
    assert checked == R


def test_fp8_layer_forward():
    """Whole layer with FP8 experts (routed and shared) vs the oracle's layer with
    the FP8 expert, fed the GPU's routing decision."""
    w = _fp8_layer_case()
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
                          expert_ffn=O.swiglu_ffn_fp8)
    assert rel_err(f64(lay.y[:w.T]), out["y"]) < TOL_FP8


def test_fp8_deepseek_v3_sampled_tokens():
    """The DeepSeek-V3-shaped FP8 layer at full size, checked on sampled tokens."""
    w = WORKLOADS["deepseek_v3_fp8"]
    inp = make_inputs(w, "cuda")
    lay = MoELayer(w, inp, "cuda", update_bias=False)
    lay.forward(inp["x"])
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    toks = np.random.default_rng(1).choice(w.T, size=8, replace=False)
    cfg = oracle_cfg(w)
    get = expert_weights_fn(inp)
    idx, wts = i64(lay.topk_idx), f64(lay.topk_w)
    x64 = f64(inp["x"])
    ws = shared_weights(inp)
    y_gpu = f64(lay.y[torch.tensor(toks, device="cuda")])
    # one oracle FP8 expert call per distinct expert (its weights quantised once)
    y_ref = O.swiglu_ffn_fp8(x64[toks], *ws)
    by_expert = {}
    for i, t in enumerate(toks):
        for j in range(w.k):
            by_expert.setdefault(int(idx[t, j]), []).append((i, j))
    for e, uses in by_expert.items():
        rows = [i for i, _ in uses]
        ye = O.swiglu_ffn_fp8(x64[toks[rows]], *get(e))
        for r_i, (i, j) in enumerate(uses):
            y_ref[i] += wts[toks[i], j] * ye[r_i]
    for i, t in enumerate(toks):
        assert rel_err(y_gpu[i], y_ref[i]) < TOL_FP8, (t, rel_err(y_gpu[i], y_ref[i]))
    assert cfg.top_k == w.k
