"""Seeded synthetic inputs for the MoE layer workloads.

This module holds only workload shapes and random-number recipes: no step of the
layer's arithmetic.  It is the one module that both the CUDA path's callers and
the oracle tests draw inputs from.

Recipe (seed 0 unless stated): tensors drawn in the fixed order x, W_g, b, W1, W3,
W2, then the shared experts' W1, W3, W2, from one torch.Generator on the target
device; x ~ N(0, 1); every weight ~ N(0, 1/fan_in) with fan_in = d for W_g, W1, W3
and fan_in = f for W2; the selection bias b ~ N(0, 0.01) read as variance 0.01
(std 0.1); expert weights are drawn 8 experts at a time (to bound the fp32
temporary) and rounded to the storage dtype.  The Switch-style workload adds the
fixed per-expert logit offset o[e] = -1.1 * ln(e + 1), the log of an unnormalised
Zipf(s = 1.1) weight, so expert 0 is the hottest.
With the shared-expert sink, W_g has one extra (last) row scoring the shared expert.
FP8 workloads draw the same bf16 tensors; the layer quantises them.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    N: int
    k: int
    f: int
    n_shared: int = 0
    f_shared: int = 0
    score: str = "softmax"              # "softmax" | "sigmoid"
    n_groups: int = 1
    topk_groups: int = 1
    group_topn: int = 2
    capacity: str = "dropless"          # "dropless" | "ceil_cf_T_over_N" | "floor_cf_k_T_over_N"
    cf: float = 1.0
    dtype: str = "bf16"                 # storage / compute type of x and experts
    bias_std: float = 0.0               # > 0: selection bias drawn with this std
    zipf_s: float = 0.0                 # > 0: per-expert logit offset -s ln(e+1)
    alpha: float = 0.01                 # aux-loss coefficient reported in the stats
    z_coef: float = 1e-3                # z-loss coefficient reported in the stats
    bias_rate: float = 1e-3             # aux-loss-free bias update step
    renorm: bool = True
    shared_sink: bool = False           # the (single) shared expert joins the weight normalisation
    expert_choice: bool = False         # experts pick their top-C tokens (C = ceil(cf k T / N))
    fp8: bool = False                   # expert matmuls on E4M3 codes with fine-grained block scales
    mxfp8: bool = False                 # expert matmuls in MXFP8 (E4M3, E8M0 scale per 32 along K)
    nvfp4: bool = False                 # expert matmuls in NVFP4 (E2M1, E4M3 scale per 16, fp32 per tensor)

    def with_tokens(self, T: int) -> "Workload":
        return replace(self, T=T)


WORKLOADS = {
    "tiny_top2_fp32": Workload("tiny_top2_fp32", T=256, d=128, N=8, k=2, f=256,
                               capacity="ceil_cf_T_over_N", cf=1.25, dtype="fp32"),
    "mixtral_8x7b": Workload("mixtral_8x7b", T=4096, d=4096, N=8, k=2, f=14336),
    "deepseekmoe_16b": Workload("deepseekmoe_16b", T=8192, d=2048, N=64, k=6, f=1408,
                                n_shared=2, f_shared=1408),
    "deepseek_v3": Workload("deepseek_v3", T=16384, d=7168, N=256, k=8, f=2048, n_shared=1,
                            f_shared=2048, score="sigmoid", n_groups=8, topk_groups=4,
                            group_topn=2, bias_std=0.1),
    "switch_skewed": Workload("switch_skewed", T=65536, d=1024, N=128, k=1, f=4096,
                              capacity="ceil_cf_T_over_N", cf=1.0, zipf_s=1.1),
    # expert-choice routing on the DeepSeekMoE-16B shape: k = 6 experts per token on
    # average, so each of the 64 experts takes C = 768 tokens
    "ec_deepseekmoe_16b": Workload("ec_deepseekmoe_16b", T=8192, d=2048, N=64, k=6, f=1408,
                                   n_shared=2, f_shared=1408, expert_choice=True),
    # the DeepSeek-V3 shape with every expert matmul (routed and shared) in FP8: bf16
    # x and weights drawn as above, quantised by the layer (1 x 128 / 128 x 128 blocks)
    "deepseek_v3_fp8": Workload("deepseek_v3_fp8", T=16384, d=7168, N=256, k=8, f=2048, n_shared=1,
                                f_shared=2048, score="sigmoid", n_groups=8, topk_groups=4,
                                group_topn=2, bias_std=0.1, fp8=True),
    # the same with MXFP8 experts (scales applied by the tensor cores)
    "deepseek_v3_mxfp8": Workload("deepseek_v3_mxfp8", T=16384, d=7168, N=256, k=8, f=2048, n_shared=1,
                                  f_shared=2048, score="sigmoid", n_groups=8, topk_groups=4,
                                  group_topn=2, bias_std=0.1, mxfp8=True),
    # the same with NVFP4 experts (block scales applied by the tensor cores)
    "deepseek_v3_nvfp4": Workload("deepseek_v3_nvfp4", T=16384, d=7168, N=256, k=8, f=2048, n_shared=1,
                                  f_shared=2048, score="sigmoid", n_groups=8, topk_groups=4,
                                  group_topn=2, bias_std=0.1, nvfp4=True),
}


def torch_dtype(w: Workload) -> torch.dtype:
    return torch.float32 if w.dtype == "fp32" else torch.bfloat16


def zipf_offset(N: int, s: float) -> torch.Tensor:
    return torch.tensor([-s * math.log(e + 1.0) for e in range(N)], dtype=torch.float32)


def make_inputs(w: Workload, device="cuda", seed: int = 0, experts: bool = True) -> dict:
    """All tensors of one workload, drawn in the fixed order of the recipe."""
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    dt = torch_dtype(w)

    def randn(shape, std):
        return (torch.randn(shape, generator=g, device=dev, dtype=torch.float32) * std)

    out = {"x": randn((w.T, w.d), 1.0).to(dt).contiguous(),
           "w_gate": randn((w.N + (1 if w.shared_sink else 0), w.d), 1.0 / math.sqrt(w.d)).contiguous()}
    out["bias"] = randn((w.N,), w.bias_std).contiguous() if w.bias_std > 0 else None
    out["logit_offset"] = zipf_offset(w.N, w.zipf_s).to(dev) if w.zipf_s > 0 else None
    if not experts:
        return out

    def expert_stack(n, rows, cols, std):
        t = torch.empty((n, rows, cols), dtype=dt, device=dev)
        for e0 in range(0, n, 8):
            e1 = min(n, e0 + 8)
            t[e0:e1] = randn((e1 - e0, rows, cols), std).to(dt)
        return t

    out["w1"] = expert_stack(w.N, w.f, w.d, 1.0 / math.sqrt(w.d))
    out["w3"] = expert_stack(w.N, w.f, w.d, 1.0 / math.sqrt(w.d))
    out["w2"] = expert_stack(w.N, w.d, w.f, 1.0 / math.sqrt(w.f))
    if w.n_shared > 0:
        fs = w.n_shared * w.f_shared
        # the shared experts' matrices concatenated along the hidden dimension
        out["ws1"] = expert_stack(1, fs, w.d, 1.0 / math.sqrt(w.d))[0].contiguous()
        out["ws3"] = expert_stack(1, fs, w.d, 1.0 / math.sqrt(w.d))[0].contiguous()
        out["ws2"] = expert_stack(1, w.d, fs, 1.0 / math.sqrt(w.f_shared))[0].contiguous()
    return out


def random_routing(T: int, N: int, k: int, device="cpu", seed: int = 0,
                   hot: Optional[int] = None) -> torch.Tensor:
    """k distinct experts per token drawn uniformly (or all tokens forced to pick
    expert `hot` first), for permutation tests that bypass the router."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    idx = torch.argsort(torch.rand((T, N), generator=g), dim=1)[:, :k].to(torch.int32)
    if hot is not None:
        for t in range(T):
            row = idx[t].tolist()
            if hot in row:
                row.remove(hot)
            else:
                row.pop()
            idx[t] = torch.tensor([hot] + row, dtype=torch.int32)
    return idx.to(device)
