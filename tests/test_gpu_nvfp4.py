"""GPU-vs-oracle parity of the NVFP4 expert path, through the C ABI.

Quantisation (packed E2M1 codes, E4M3 block-scale bytes, fp32 tensor scales) is
compared bit for bit: every step is an fp32 operation both sides take in the same
order.  h is re-quantised from the GPU's GEMM and the oracle's fp64 one, so it is
checked by the fraction of equal scales and codes and by the error bound of one
E2M1 step; y against the oracle's down projection of the GPU's own h, and against
the oracle's NVFP4 expert end to end.
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
from tests.test_gpu_fp8 import decode_e4m3

pytestmark = pytest.mark.gpu

TOL_NV_SAME_H = 5e-3    # y vs the oracle's down projection of the GPU's own h codes
# y vs the oracle's NVFP4 expert end to end.  An h element whose GPU and fp64 values
# straddle an E2M1 rounding boundary would move by a whole step (up to a third of its
# value); measured: no such flips on these cases (h codes equal), y within 2.8e-3 per
# group and 4.6e-3 for the layer, so the bound leaves room for a few flips only
TOL_NV = 2e-2


def decode_e2m1(packed: np.ndarray) -> np.ndarray:
    """Packed bytes [R, C / 2] -> values [R, C]: element 2i in the low nibble; each
    nibble is sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0; exponent 0 is
    subnormal (m / 2)."""
    p = np.asarray(packed, np.int64)
    nib = np.stack([p & 0xF, p >> 4], axis=-1).reshape(p.shape[0], -1)
    sign = np.where(nib & 8, -1.0, 1.0)
    e = (nib >> 1) & 3
    m = nib & 1
    return sign * np.where(e == 0, m * 0.5, (1.0 + m / 2.0) * 2.0 ** (e - 1))


def nv_scales_rowmajor(sf, rows: int, cols: int, offsets=None) -> np.ndarray:
    """Tile atoms -> numpy [rows, cols / 16] scale bytes (rows grouped by `offsets`, a
    sequence of G + 1 row offsets, or one plain group)."""
    a = sf.cpu().numpy() if hasattr(sf, "cpu") else np.asarray(sf)
    nch = cols // 64
    off = [0, rows] if offsets is None else [int(o) for o in offsets]
    out = np.zeros((rows, cols // 16), np.uint8)
    tile = 0
    m = np.arange(128)
    pos = 16 * (m % 32) + 4 * (m // 32)
    for g in range(len(off) - 1):
        for r0 in range(off[g], off[g + 1], 128):
            n = min(128, off[g + 1] - r0)
            for c in range(nch):
                atom = a[(tile * nch + c) * 512:(tile * nch + c + 1) * 512]
                for j in range(4):
                    out[r0:r0 + n, 4 * c + j] = atom[pos[:n] + j]
            tile += 1
    return out


def gpu_nv(x: torch.Tensor, tensor_rows: int = 0):
    R, C = x.shape
    q = torch.empty(R, C // 2, dtype=torch.uint8, device="cuda")
    sf = L.nv_scales(R, C, "cuda")
    g = torch.empty(max(R // tensor_rows, 1) if tensor_rows else 1, dtype=torch.float32, device="cuda")
    L.moe_quantize_nvfp4(x, q, sf, g if tensor_rows else None, tensor_rows=tensor_rows)
    return q, sf, g


def deq_nv(q, sf, g_rows=None, offsets=None) -> np.ndarray:
    """Dequantised GPU rows; g_rows: per-row tensor scale (None: 1)."""
    R = q.shape[0]
    C = 2 * q.shape[1]
    b = decode_e4m3(nv_scales_rowmajor(sf, R, C, offsets))
    v = decode_e2m1(q.cpu().numpy()) * np.repeat(b, 16, axis=1)
    return v if g_rows is None else v * np.asarray(g_rows, np.float64)[:, None]


def test_nv_quantize_bit_exact_unit_scale():
    gen = torch.Generator(device="cuda").manual_seed(11)
    R, C = 300, 640
    x = torch.randn(R, C, generator=gen, device="cuda") * torch.exp2(
        torch.randint(-8, 8, (R, 1), generator=gen, device="cuda").float())
    x[3, :16] = 0.0                                     # an all-zero block: scale 0, codes 0
    x[4, 64:80] = 3.0                                   # amax / 6 = 0.5 exactly: codes 6
    x[5, 96:112] = 3000.0                               # the block scale saturates at 448
    x[6, 7] = 1e-4                                      # a tiny block element
    x[7, 128:144] = 2.0 ** -12                          # block scale underflows to 0
    xb = x.to(torch.bfloat16)
    q, sf, _ = gpu_nv(xb)
    torch.cuda.synchronize()
    q_ref, b_ref = O.quantize_nvfp4(f64(xb))
    assert np.array_equal(decode_e4m3(nv_scales_rowmajor(sf, R, C)), b_ref)
    assert np.array_equal(decode_e2m1(q.cpu().numpy()), q_ref)


def test_nv_quantize_bit_exact_tensor_scales():
    """Weights: one tensor scale per `tensor_rows` rows (an expert matrix)."""
    gen = torch.Generator(device="cuda").manual_seed(13)
    E, rows, C = 3, 256, 512
    w = (torch.randn(E, rows, C, generator=gen, device="cuda") * 0.02).to(torch.bfloat16)
    w[1] *= 40                                          # experts of different ranges
    m = w.reshape(-1, C)
    q, sf, g = gpu_nv(m, tensor_rows=rows)
    torch.cuda.synchronize()
    for e in range(E):
        we = f64(w[e])
        ge = O.nvfp4_tensor_scale(we)
        assert np.float32(g[e].item()) == ge
        q_ref, b_ref = O.quantize_nvfp4(we, ge)
        lo, hi = e * rows, (e + 1) * rows
        assert np.array_equal(decode_e4m3(nv_scales_rowmajor(sf, E * rows, C))[lo:hi], b_ref)
        assert np.array_equal(decode_e2m1(q[lo:hi].cpu().numpy()), q_ref)


def _nv_layer_case():
    return replace(WORKLOADS["deepseekmoe_16b"], name="dsmoe_nv_small", T=777, d=512, N=16, k=6,
                   f=256, n_shared=1, f_shared=512, nvfp4=True)


def test_permute_nvfp4_rows_bit_exact():
    w = _nv_layer_case()
    inp = make_inputs(w, "cuda")
    lay = MoELayer(w, inp, "cuda", update_bias=False)
    c = lay.cfg
    L.moe_route(c, inp["x"], inp["w_gate"], None, inp.get("bias"), lay.topk_idx, lay.topk_w, lay.lse,
                lay.p_partial, lay.margin, lay.ws)
    L.moe_permute(c, None, lay.topk_idx, lay.counts, lay.offsets, lay.row_of_slot, lay.token_of_row, None,
                  lay.n_dropped, lay.ws)
    L.moe_permute_nvfp4(c, inp["x"], lay.topk_idx, lay.row_of_slot, lay.offsets, lay.xq_perm, lay.xs_perm,
                        lay.xq, lay.xs)
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    q_ref, b_ref = O.quantize_nvfp4(f64(inp["x"]))
    R = int(lay.offsets[-1].item())
    tor = i64(lay.token_of_row)[:R]
    off = i64(lay.offsets)
    assert np.array_equal(decode_e2m1(lay.xq_perm[:R].cpu().numpy()), q_ref[tor])
    assert np.array_equal(decode_e4m3(nv_scales_rowmajor(lay.xs_perm, R, w.d, off)), b_ref[tor])
    assert np.array_equal(decode_e2m1(lay.xq[:w.T].cpu().numpy()), q_ref)
    assert np.array_equal(decode_e4m3(nv_scales_rowmajor(lay.xs, w.T, w.d)), b_ref)


@pytest.mark.parametrize("d,f,sizes", [
    (256, 256, [0, 1, 130, 257, 77]),        # empty and 1-row groups, ragged tails
    (512, 512, [128, 0, 0, 300]),            # 2 N tiles of y, 4 of h
    (7168, 2048, [5, 0, 190]),                # the DeepSeek-V3 expert shape
])
def test_grouped_ffn_nvfp4(d, f, sizes):
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
    xq = torch.empty(rows_cap, d // 2, dtype=torch.uint8, device="cuda")
    xsf = L.nv_scales(rows_cap, d, "cuda", G)
    nch = d // 64
    tile = 0
    for g in range(G):
        n = int(off[g + 1] - off[g])
        if n == 0:
            continue
        qg, sg, _ = gpu_nv(x[off[g]:off[g + 1]])
        xq[off[g]:off[g + 1]] = qg
        nt = (n + 127) // 128
        xsf[tile * nch * 512:(tile + nt) * nch * 512] = sg[:nt * nch * 512]
        tile += nt
    (w1q, w1sf, g1), (w3q, w3sf, g3) = (gpu_nv(t.reshape(-1, d), tensor_rows=f) for t in (w1, w3))
    w2q, w2sf, g2 = gpu_nv(w2.reshape(-1, f), tensor_rows=d)
    hq = torch.zeros(rows_cap, f // 2, dtype=torch.uint8, device="cuda")
    hsf = L.nv_scales(rows_cap, f, "cuda", G).zero_()
    y = torch.full((rows_cap, d), 7.0, dtype=torch.bfloat16, device="cuda")
    cfg = make_config(replace(WORKLOADS["deepseek_v3"], d=d, T=R))
    L.moe_grouped_ffn_nvfp4(cfg, xq, xsf, rows_cap, torch.tensor(off, device="cuda"), G, w1q, w1sf, g1, w3q,
                            w3sf, g3, w2q, w2sf, g2, f, hq, hsf, y)
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    assert torch.all(y[R:] == 7.0)
    x64 = f64(x)
    h_gpu = deq_nv(hq[:R], hsf, None, off)
    b_h = decode_e4m3(nv_scales_rowmajor(hsf, R, f, off))
    y_gpu = f64(y)
    checked = 0
    for g in range(G):
        lo, hi = off[g], off[g + 1]
        if hi == lo:
            continue
        xd = O.dequantize_nvfp4(*O.quantize_nvfp4(x64[lo:hi]))

        def wq(t):
            ge = O.nvfp4_tensor_scale(t)
            return O.dequantize_nvfp4(*O.quantize_nvfp4(t, ge), ge)

        wd = [wq(f64(t[g])) for t in (w1, w3, w2)]
        h_ref = O.silu(xd @ wd[0].T) * (xd @ wd[1].T)
        q_ref, b_ref = O.quantize_nvfp4(h_ref)
        same_b = np.mean(b_h[lo:hi] == b_ref)
        # the oracle's rounding of h_ref under the GPU's own block scales
        s_gpu = np.repeat(b_h[lo:hi], 16, axis=1)
        with np.errstate(divide="ignore", invalid="ignore"):
            q_same = np.where(s_gpu > 0, s_gpu * O.round_e2m1((h_ref / s_gpu).astype(np.float32)), 0.0)
        same = np.mean(h_gpu[lo:hi] == q_same)
        print(f"group {g}: rows {hi - lo}, block scales equal {same_b:.4f}, values equal {same:.4f}")
        assert same_b >= 0.97 and same >= 0.95, (same_b, same)
        # every element within one E2M1 step (at its block's scale) of the exact h
        assert np.all(np.abs(h_gpu[lo:hi] - h_ref) <= 2.0 * s_gpu + 1e-6 * np.abs(h_ref))
        assert rel_err(y_gpu[lo:hi], h_gpu[lo:hi] @ wd[2].T) < TOL_NV_SAME_H
        y_ref = O.swiglu_ffn_nvfp4(x64[lo:hi], f64(w1[g]), f64(w3[g]), f64(w2[g]))
        print(f"group {g}: y vs the oracle's NVFP4 expert {rel_err(y_gpu[lo:hi], y_ref):.3e}")
        assert rel_err(y_gpu[lo:hi], y_ref) < TOL_NV
        checked += hi - lo
    assert checked == R


def test_nvfp4_layer_forward():
    w = _nv_layer_case()
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
                          expert_ffn=O.swiglu_ffn_nvfp4)
    err = rel_err(f64(lay.y[:w.T]), out["y"])
    print(f"NVFP4 layer: y vs oracle {err:.3e}")
    assert err < TOL_NV


def test_nvfp4_deepseek_v3_sampled_tokens():
    """The DeepSeek-V3-shaped layer with NVFP4 experts, at full size: sampled tokens
    against the oracle's NVFP4 experts under the GPU's routing."""
    w = WORKLOADS["deepseek_v3_nvfp4"]
    inp = make_inputs(w, "cuda")
    lay = MoELayer(w, inp, "cuda", update_bias=False)
    lay.forward(inp["x"])
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    toks = np.random.default_rng(3).choice(w.T, size=4, replace=False)
    get = expert_weights_fn(inp)
    idx, wts = i64(lay.topk_idx), f64(lay.topk_w)
    x64 = f64(inp["x"])
    y_gpu = f64(lay.y[torch.tensor(toks, device="cuda")])
    y_ref = O.swiglu_ffn_nvfp4(x64[toks], *shared_weights(inp))
    by_expert = {}
    for i, t in enumerate(toks):
        for j in range(w.k):
            by_expert.setdefault(int(idx[t, j]), []).append((i, j))
    for e, uses in by_expert.items():
        ye = O.swiglu_ffn_nvfp4(x64[toks[[i for i, _ in uses]]], *get(e))
        for r_i, (i, j) in enumerate(uses):
            y_ref[i] += wts[toks[i], j] * ye[r_i]
    for i, t in enumerate(toks):
        assert rel_err(y_gpu[i], y_ref[i]) < TOL_NV, (t, rel_err(y_gpu[i], y_ref[i]))
