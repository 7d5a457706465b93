"""Helpers shared by the GPU parity tests: oracle configs, conversions, error norms."""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_21_b200.synth import Workload

# Tolerances (max |a - b| / max |b| per output tensor): the layer's stated bar.
TOL_BF16 = 2e-2
TOL_F32 = 1e-4
TOL_STATS = 1e-5
NEAR_TIE = 1e-4


def oracle_cfg(w: Workload) -> O.OracleConfig:
    cap = {"dropless": O.CAP_DROPLESS, "ceil_cf_T_over_N": O.CAP_CEIL_CF_T_OVER_N,
           "floor_cf_k_T_over_N": O.CAP_CF_K_T_OVER_N_FLOOR}[w.capacity]
    return O.OracleConfig(n_experts=w.N, top_k=w.k,
                          score_fn=O.SIGMOID if w.score == "sigmoid" else O.SOFTMAX,
                          renorm=w.renorm, n_groups=w.n_groups, topk_groups=w.topk_groups,
                          group_score_topn=w.group_topn, capacity_mode=cap,
                          capacity_factor=w.cf)


def f64(t) -> np.ndarray:
    if t is None:
        return None
    return t.detach().cpu().to(torch.float64).numpy()


def i64(t) -> np.ndarray:
    return t.detach().cpu().to(torch.int64).numpy()


def rel_err(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    denom = np.max(np.abs(b))
    return float(np.max(np.abs(a - b)) / denom) if denom > 0 else float(np.max(np.abs(a - b)))


def tol_for(w: Workload) -> float:
    return TOL_F32 if w.dtype == "fp32" else TOL_BF16


def expert_weights_fn(inp: dict):
    """Oracle-side view of expert e's (w1, w3, w2), widened to fp64 on demand."""
    def get(e):
        return f64(inp["w1"][e]), f64(inp["w3"][e]), f64(inp["w2"][e])
    return get


def shared_weights(inp: dict):
    if "ws1" not in inp:
        return None
    return f64(inp["ws1"]), f64(inp["ws3"]), f64(inp["ws2"])


def mx_scales_rowmajor(sf, rows: int, cols: int, offsets=None):
    """Tile atoms -> numpy [rows, cols / 32] scale bytes (rows grouped by `offsets`, a
    sequence of G + 1 row offsets, or one plain group)."""
    a = sf.cpu().numpy() if hasattr(sf, "cpu") else np.asarray(sf)
    nkb = cols // 128
    off = [0, rows] if offsets is None else [int(o) for o in offsets]
    out = np.zeros((rows, cols // 32), np.uint8)
    tile = 0
    m = np.arange(128)
    pos = 16 * (m % 32) + 4 * (m // 32)
    for g in range(len(off) - 1):
        for r0 in range(off[g], off[g + 1], 128):
            n = min(128, off[g + 1] - r0)
            for kb in range(nkb):
                atom = a[(tile * nkb + kb) * 512:(tile * nkb + kb + 1) * 512]
                for j in range(4):
                    out[r0:r0 + n, 4 * kb + j] = atom[pos[:n] + j]
            tile += 1
    return out
