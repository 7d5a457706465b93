"""Edge cases of the FP8 and MXFP8 layers against the oracle: capacity drop with
skewed routing, fewer tokens than one tile, no tokens at all, and every token
routed to one expert."""
from __future__ import annotations

from dataclasses import replace

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_21_b200 import _lib as L
from sparse_mixture_experts_21_b200.layer import MoELayer
from sparse_mixture_experts_21_b200.synth import WORKLOADS, make_inputs
from tests.parity_util import NEAR_TIE, expert_weights_fn, f64, i64, oracle_cfg, rel_err, shared_weights

pytestmark = pytest.mark.gpu

TOL = 2e-2
MODES = {"fp8": (dict(fp8=True), O.swiglu_ffn_fp8), "mxfp8": (dict(mxfp8=True), O.swiglu_ffn_mxfp8)}


def _layer(w):
    inp = make_inputs(w, "cuda")
    lay = MoELayer(w, inp, "cuda", update_bias=False)
    lay.forward(inp["x"])
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    return lay, inp


def _oracle_y(w, lay, inp, ffn):
    return O.layer_forward(f64(inp["x"]), None, oracle_cfg(w), expert_weights_fn(inp), shared_weights(inp),
                           routing={"idx": i64(lay.topk_idx), "w": f64(lay.topk_w)}, expert_ffn=ffn)


@pytest.mark.parametrize("mode", MODES)
def test_capacity_drop_skewed(mode):
    """Switch-style top-1 with capacity cf = 1 and a Zipf offset: many tokens dropped;
    their output rows are zero and the kept ones match the oracle."""
    flags, ffn = MODES[mode]
    w = replace(WORKLOADS["switch_skewed"], name=f"switch_{mode}_small", T=900, d=256, N=8, f=384, **flags)
    lay, inp = _layer(w)
    out = _oracle_y(w, lay, inp, ffn)
    dropped = i64(lay.row_of_slot)[:, 0] < 0
    assert dropped.sum() > 100
    assert int(lay.n_dropped[1].item()) == int(dropped.sum())
    y = f64(lay.y[:w.T])
    assert np.all(y[dropped] == 0.0)
    assert rel_err(y, out["y"]) < TOL


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("T", [1, 3, 129])
def test_few_tokens(mode, T):
    flags, ffn = MODES[mode]
    w = replace(WORKLOADS["deepseekmoe_16b"], name=f"ds_{mode}_T{T}", T=T, d=256, N=16, k=6, f=256,
                n_shared=1, f_shared=256, **flags)
    lay, inp = _layer(w)
    r = O.route(f64(inp["x"]), f64(inp["w_gate"]), oracle_cfg(w))
    clear = r["margin"] >= NEAR_TIE
    assert np.array_equal(i64(lay.topk_idx)[clear], r["idx"][clear])
    assert rel_err(f64(lay.y[:w.T]), _oracle_y(w, lay, inp, ffn)["y"]) < TOL


@pytest.mark.parametrize("mode", MODES)
def test_no_tokens(mode):
    flags, _ = MODES[mode]
    w = replace(WORKLOADS["deepseekmoe_16b"], name=f"ds_{mode}_T0", T=0, d=256, N=16, k=6, f=256,
                n_shared=1, f_shared=256, **flags)
    lay, inp = _layer(w)
    assert int(lay.offsets[-1].item()) == 0
    assert torch.all(lay.counts == 0)


@pytest.mark.parametrize("mode", MODES)
def test_all_tokens_one_expert(mode):
    """A logit offset that makes expert 3 every token's first choice: one group of T
    rows (several tiles, ragged tail) and k - 1 other groups."""
    flags, ffn = MODES[mode]
    w = replace(WORKLOADS["mixtral_8x7b"], name=f"mix_{mode}_hot", T=333, d=256, f=384, **flags)
    inp = make_inputs(w, "cuda")
    off = torch.zeros(w.N, device="cuda")
    off[3] = 50.0
    inp["logit_offset"] = off
    lay = MoELayer(w, inp, "cuda", update_bias=False)
    lay.forward(inp["x"])
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    counts = i64(lay.counts)
    assert counts[3] == w.T
    out = O.layer_forward(f64(inp["x"]), None, oracle_cfg(w), expert_weights_fn(inp), None,
                          routing={"idx": i64(lay.topk_idx), "w": f64(lay.topk_w)}, expert_ffn=ffn)
    assert rel_err(f64(lay.y[:w.T]), out["y"]) < TOL


@pytest.mark.parametrize("mode", ["fp8", "mxfp8", "nvfp4"])
@pytest.mark.parametrize("T", [777, 100])
def test_shared_expert_on_side_stream_equals_main_stream(mode, T):
    """Low-precision shared experts quantised and computed on a side stream during route
    and permute give the same output bit for bit as after the routed experts on the main
    stream (whose input codes the quantising scatter writes)."""
    flags = {"fp8": dict(fp8=True), "mxfp8": dict(mxfp8=True), "nvfp4": dict(nvfp4=True)}[mode]
    w = replace(WORKLOADS["deepseekmoe_16b"], name=f"dsmoe_{mode}_small", T=T, d=512, N=16, k=6, f=256,
                n_shared=1, f_shared=512, **flags)
    inp = make_inputs(w, "cuda")
    a = MoELayer(w, inp, "cuda", update_bias=False, overlap_shared=False)
    b = MoELayer(w, inp, "cuda", update_bias=False, overlap_shared=True)
    assert b.overlap_shared and not a.overlap_shared
    ya = a.forward(inp["x"]).clone()
    for _ in range(2):
        yb = b.forward(inp["x"]).clone()
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    assert torch.equal(ya, yb)
    assert torch.equal(a.ys[:T], b.ys[:T])
