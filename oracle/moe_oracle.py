"""Plain, slow, double-precision CPU oracle of the sparse MoE FFN layer forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it.  It shares no code with the CUDA library and never reads
anything that the CUDA library produced, except where a test deliberately
cross-feeds the GPU's routing decisions into the oracle's permutation step.

Every step follows the source pages in their order and notation; each function
names the page and section it restates.  Page tags used below:

  [Practice]  "混合专家模型（MoE）架构实战：路由策略、负载均衡与工程实现"
              (deepseekmodel.com blog)
  [Compass]   "llm-compass: MoE" (brenchcc.github.io, architecture/moe)
  [Taste]     "MoE common taste in open models" (r00kie-liu.github.io)
  [Landscape] "MoE landscape" (cyk1337 paper-daily topic page)
  [History]   "MoE 的工业进化：从 1.6 万亿的 Switch Transformer 到 2.8 万亿的 Kimi K3"
              (alishangtian.com)

Where the pages are silent or disagree, the reading taken is stated at the
function.  All arithmetic is float64; integer decisions (top-k, capacity,
positions) are made on float64 scores.  Library primitives used as single steps:
``numpy.matmul``, ``numpy.argsort(kind="stable")``, ``numpy.exp``/``log``.

Pinned by ``tests/test_oracle_pins.py`` (worked example, brute-force top-k, closed
forms, invariants); no function here is "parity unpinned".
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional, Sequence

import numpy as np

SOFTMAX = "softmax"
SIGMOID = "sigmoid"

CAP_DROPLESS = "dropless"
CAP_CEIL_CF_T_OVER_N = "ceil_cf_T_over_N"          # north-star / [Compass] form
CAP_CF_K_T_OVER_N_FLOOR = "floor_cf_k_T_over_N"    # [Practice] code form


@dataclass
class OracleConfig:
    """Shape and routing options of one MoE layer (oracle-side copy)."""

    n_experts: int
    top_k: int
    score_fn: str = SOFTMAX
    renorm: bool = True
    n_groups: int = 1            # 1: no group-limited pre-selection
    topk_groups: int = 1
    group_score_topn: int = 2
    capacity_mode: str = CAP_DROPLESS
    capacity_factor: float = 1.0


# ---------------------------------------------------------------------------
# 1. Router GEMM
# ---------------------------------------------------------------------------
def router_logits(x: np.ndarray, w_gate: np.ndarray,
                  logit_offset: Optional[np.ndarray] = None) -> np.ndarray:
    """z[t, e] = sum_d x[t, d] * Wg[e, d]  (+ o[e] when a per-expert offset is given).

    [Practice] section "路由的数学形式": the gate is a bias-free linear layer over the
    flattened [T, D] tokens.  [Compass] section "稀疏门控与 Top-k 路由": affinity x·W_g.
    The optional offset o[e] is the synthetic Zipf skew of the Switch-style stress
    workload, added to the logits (a workload input, not a router bias).
    """
    z = np.asarray(x, dtype=np.float64) @ np.asarray(w_gate, dtype=np.float64).T
    if logit_offset is not None:
        z = z + np.asarray(logit_offset, dtype=np.float64)[None, :]
    return z


# ---------------------------------------------------------------------------
# 2. Affinity
# ---------------------------------------------------------------------------
def softmax(z: np.ndarray) -> np.ndarray:
    """Row softmax exp(z - max) / sum exp(z - max)  ([Practice] "路由的数学形式")."""
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    return e / e.sum(axis=1, keepdims=True)


def sigmoid(z: np.ndarray) -> np.ndarray:
    """Independent per-expert score 1 / (1 + exp(-z))  ([Taste] section 7)."""
    return 1.0 / (1.0 + np.exp(-z))


def logsumexp(z: np.ndarray) -> np.ndarray:
    """log sum_e exp(z[t, e]) per token, used by the router z-loss."""
    m = z.max(axis=1)
    return m + np.log(np.exp(z - m[:, None]).sum(axis=1))


def affinity(z: np.ndarray, score_fn: str) -> np.ndarray:
    if score_fn == SOFTMAX:
        return softmax(z)
    if score_fn == SIGMOID:
        return sigmoid(z)
    raise ValueError(score_fn)


# ---------------------------------------------------------------------------
# 3. Selection score with the choice-only bias
# ---------------------------------------------------------------------------
def selection_scores(s: np.ndarray, bias: Optional[np.ndarray]) -> np.ndarray:
    """q = s + b: the bias is added to the affinity for choosing only.

    [Compass] section "负载均衡：从 aux loss 到 aux-loss-free": Top-k({s_i + b_i}), with
    the gate weights still proportional to the raw s_i.  [Practice] class
    BiasBalancedRouter adds the bias to the softmax probabilities, not the logits.
    """
    if bias is None:
        return s.copy()
    return s + np.asarray(bias, dtype=np.float64)[None, :]


# ---------------------------------------------------------------------------
# 4. Group-limited pre-selection (reading: the pages give no formula)
# ---------------------------------------------------------------------------
def group_scores(q: np.ndarray, n_groups: int, topn: int) -> np.ndarray:
    """Score of each contiguous expert group = sum of its `topn` largest q.

    [History] part 四 and [Practice] "负载均衡损失" name node-limited routing without
    a formula; reading: experts split into n_groups contiguous groups of N/n_groups,
    scored by the sum of their top-`topn` selection scores (topn = 1 gives max).
    """
    T, N = q.shape
    gs = N // n_groups
    qg = q.reshape(T, n_groups, gs)
    top = -np.sort(-qg, axis=2)[:, :, :topn]
    return top.sum(axis=2)


def eligible_mask(q: np.ndarray, cfg: OracleConfig) -> tuple[np.ndarray, np.ndarray]:
    """Experts a token may pick after keeping its `topk_groups` best groups.

    Returns (mask [T, N] bool, group_margin [T]).  Group ties: lower group index wins.
    group_margin is the score of the last kept group minus the best dropped group
    (+inf when no group is dropped).
    """
    T, N = q.shape
    if cfg.n_groups <= 1:
        return np.ones((T, N), dtype=bool), np.full(T, np.inf)
    gsc = group_scores(q, cfg.n_groups, cfg.group_score_topn)
    order = np.argsort(-gsc, axis=1, kind="stable")          # descending, lower index first on ties
    kept = order[:, : cfg.topk_groups]
    gs = N // cfg.n_groups
    mask = np.zeros((T, N), dtype=bool)
    for t in range(T):
        for g in kept[t]:
            mask[t, g * gs:(g + 1) * gs] = True
    if cfg.topk_groups < cfg.n_groups:
        last = np.take_along_axis(gsc, order[:, cfg.topk_groups - 1:cfg.topk_groups], axis=1)[:, 0]
        first_out = np.take_along_axis(gsc, order[:, cfg.topk_groups:cfg.topk_groups + 1], axis=1)[:, 0]
        gmargin = last - first_out
    else:
        gmargin = np.full(T, np.inf)
    return mask, gmargin


# ---------------------------------------------------------------------------
# 5. Top-k
# ---------------------------------------------------------------------------
def select_topk(q: np.ndarray, k: int, mask: Optional[np.ndarray] = None
                ) -> tuple[np.ndarray, np.ndarray]:
    """The k eligible experts with the largest q, stored in descending q.

    [Practice] "路由的数学形式" (probs.topk) and [Compass] "稀疏门控与 Top-k 路由".
    Ties (pages silent): the lower expert index wins.
    Returns (idx [T, k] int64, margin [T]) where margin = q of the k-th pick minus
    the best eligible expert left out (+inf when none is left).
    """
    qq = q.copy()
    if mask is not None:
        qq[~mask] = -np.inf
    order = np.argsort(-qq, axis=1, kind="stable")
    idx = order[:, :k]
    kth = np.take_along_axis(qq, order[:, k - 1:k], axis=1)[:, 0]
    if qq.shape[1] > k:
        nxt = np.take_along_axis(qq, order[:, k:k + 1], axis=1)[:, 0]
        margin = np.where(np.isfinite(nxt), kth - nxt, np.inf)
    else:
        margin = np.full(q.shape[0], np.inf)
    return idx.astype(np.int64), margin


# ---------------------------------------------------------------------------
# 6. Gate weights
# ---------------------------------------------------------------------------
def gate_weights(s: np.ndarray, idx: np.ndarray, renorm: bool = True) -> np.ndarray:
    """w[t, j] = s[t, idx_j] / sum_j' s[t, idx_j'] (renormalised top-k weights).

    [Practice] "路由的数学形式": after top-k the k probabilities are renormalised to sum
    to one; [Compass] "负载均衡": with a bias the weights still use the raw s_i.
    renorm=False keeps w = s (a variant; no routed scaling factor on the pages).
    """
    w = np.take_along_axis(s, idx, axis=1)
    if renorm:
        w = w / w.sum(axis=1, keepdims=True)
    return w


def route(x, w_gate, cfg: OracleConfig, bias=None, logit_offset=None) -> dict:
    """Steps 1-6: logits -> affinity -> (+bias) -> group limit -> top-k -> weights."""
    z = router_logits(x, w_gate, logit_offset)
    s = affinity(z, cfg.score_fn)
    q = selection_scores(s, bias)
    mask, gmargin = eligible_mask(q, cfg)
    idx, emargin = select_topk(q, cfg.top_k, mask)
    w = gate_weights(s, idx, cfg.renorm)
    return {"logits": z, "s": s, "q": q, "idx": idx, "w": w,
            "margin": np.minimum(emargin, gmargin), "lse": logsumexp(z)}


# ---------------------------------------------------------------------------
# 7. Capacity
# ---------------------------------------------------------------------------
def capacity(cfg: OracleConfig, T: int) -> Optional[int]:
    """Per-expert capacity C, or None when dropless.

    The pages disagree ([Practice] code: max(int(cf*k*T/N), k); [Practice] prose:
    cf*k*T/N; [Compass] "容量因子与专家并行": cf*tokens/N).  Default reading:
    C = ceil(cf*T/N), evaluated as ceil((cf*T)/N) in double precision.
    """
    if cfg.capacity_mode == CAP_DROPLESS:
        return None
    N, k, cf = cfg.n_experts, cfg.top_k, cfg.capacity_factor
    if cfg.capacity_mode == CAP_CEIL_CF_T_OVER_N:
        return int(np.ceil((cf * T) / N))
    if cfg.capacity_mode == CAP_CF_K_T_OVER_N_FLOOR:
        expected = k * T / float(N)
        return max(int(expected * cf), k)
    raise ValueError(cfg.capacity_mode)


# ---------------------------------------------------------------------------
# 8. Token-order drop
# ---------------------------------------------------------------------------
def positions(idx: np.ndarray, n_experts: int) -> np.ndarray:
    """pos[t, j] = number of earlier tokens t' < t that also chose idx[t, j].

    [Practice] "路由的数学形式", third detail after the router code: the earliest
    occupants of an expert are kept ("rank == 0" wording), so drops are reproducible.
    The printed one_hot/cumsum code is garbled (it scans the k axis); the prose is
    followed.  A plain running counter over tokens in order.
    """
    T, k = idx.shape
    seen = np.zeros(n_experts, dtype=np.int64)
    pos = np.zeros((T, k), dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            pos[t, j] = seen[e]
        for j in range(k):
            seen[idx[t, j]] += 1
    return pos


# ---------------------------------------------------------------------------
# 9. Permutation into expert-contiguous rows
# ---------------------------------------------------------------------------
def permutation(idx: np.ndarray, n_experts: int, C: Optional[int]) -> dict:
    """Counts, kept counts, offsets and the slot <-> row maps.

    [Practice] "专家并行与 all-to-all": assignments are grouped stably by destination
    so one grouped GEMM covers all experts.  Rows of expert e are its kept slots in
    token order; a dropped slot (pos >= C) gets row -1 ([Practice] "容量因子、token
    dropping": a dropped token's FFN output is zero).
    """
    T, k = idx.shape
    counts = np.bincount(idx.reshape(-1), minlength=n_experts).astype(np.int64)
    pos = positions(idx, n_experts)
    keep = np.ones((T, k), dtype=bool) if C is None else pos < C
    kept = counts.copy() if C is None else np.minimum(counts, C)
    offsets = np.zeros(n_experts + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(kept)
    R = int(offsets[-1])
    row_of_slot = np.full((T, k), -1, dtype=np.int64)
    token_of_row = np.full(R, -1, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            if keep[t, j]:
                r = offsets[idx[t, j]] + pos[t, j]
                row_of_slot[t, j] = r
                token_of_row[r] = t
    dropped_slots = int(T * k - R)
    dropped_tokens = int((~keep).all(axis=1).sum())
    return {"counts": counts, "kept": kept, "offsets": offsets, "pos": pos, "keep": keep,
            "row_of_slot": row_of_slot, "token_of_row": token_of_row, "R": R,
            "dropped_slots": dropped_slots, "dropped_tokens": dropped_tokens}


def permute_rows(x: np.ndarray, token_of_row: np.ndarray) -> np.ndarray:
    """x_perm[r] = x[token_of_row[r]], with no pre-weighting.

    [Practice]'s dispatch code multiplies rows by their gate weight before the
    experts; for a nonlinear expert that contradicts [Compass]'s y = sum g_i E_i(x),
    so the weight is applied in the combine instead.
    """
    return np.asarray(x, dtype=np.float64)[token_of_row]


# ---------------------------------------------------------------------------
# 10-11. Expert FFN (SwiGLU) and shared experts
# ---------------------------------------------------------------------------
def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z / (1 + exp(-z))."""
    return z / (1.0 + np.exp(-z))


def swiglu_ffn(x_rows: np.ndarray, w1: np.ndarray, w3: np.ndarray, w2: np.ndarray) -> np.ndarray:
    """E(x) = W2 (silu(W1 x) * (W3 x)) for each row, no biases.

    The pages describe each expert as an FFN with three matrices ([Practice]
    "推理侧的路由稳定性", E x 3D^2) without defining SwiGLU; the plain reading is the
    gated form above with W1 [f, d] (gate), W3 [f, d] (up), W2 [d, f] (down).
    """
    g = x_rows @ np.asarray(w1, dtype=np.float64).T
    u = x_rows @ np.asarray(w3, dtype=np.float64).T
    h = silu(g) * u
    return h @ np.asarray(w2, dtype=np.float64).T


def swiglu_hidden(x_rows, w1, w3) -> np.ndarray:
    """h = silu(W1 x) * (W3 x), the intermediate of swiglu_ffn."""
    g = x_rows @ np.asarray(w1, dtype=np.float64).T
    u = x_rows @ np.asarray(w3, dtype=np.float64).T
    return silu(g) * u


# ---------------------------------------------------------------------------
# 12. Combine
# ---------------------------------------------------------------------------
def combine(y_rows: np.ndarray, row_of_slot: np.ndarray, w: np.ndarray,
            shared_out: Optional[np.ndarray], T: int, d: int) -> np.ndarray:
    """y[t] = ys[t] + sum over kept slots j of w[t, j] * E_{idx[t,j]}(x[t]).

    [Compass] "稀疏门控与 Top-k 路由": y = sum_{i in T} g_i E_i(x); [Practice] "共享专家":
    the always-on shared output is added.  Dropped slots contribute zero.
    """
    y = np.zeros((T, d)) if shared_out is None else np.array(shared_out, dtype=np.float64)
    for t in range(T):
        for j in range(row_of_slot.shape[1]):
            r = row_of_slot[t, j]
            if r >= 0:
                y[t] += w[t, j] * y_rows[r]
    return y


# ---------------------------------------------------------------------------
# 13. Router statistics
# ---------------------------------------------------------------------------
def normalised_affinity(s: np.ndarray, score_fn: str) -> np.ndarray:
    """s-hat: the softmax probabilities, or for sigmoid s / sum_e s (reading)."""
    if score_fn == SOFTMAX:
        return s
    return s / s.sum(axis=1, keepdims=True)


def router_stats(counts, kept, s, lse, cfg: OracleConfig, T: int,
                 dropped_slots: int, dropped_tokens: int,
                 alpha: float, z_coef: float, bias=None) -> dict:
    """f_i, P_i, aux, z-loss, usage CV, dead experts, drops, bias norm.

    [Compass] "负载均衡": L_aux = alpha * N * sum_i f_i P_i, equal to alpha under
    uniform routing ([Practice] "负载均衡损失" says 1 before scaling).  f_i is the
    share of the k*T assignments (so sum f = 1); [Practice]'s printed extra
    N*sum P^2 term contradicts its own "equals 1 when uniform" and is not used.
    z-loss: the pages name it ([History] part 五, [Landscape] §0) without a formula;
    reading = ST-MoE form mean_t (logsumexp_e z)^2.  CV: population std / mean of
    the pre-capacity counts ([Landscape] 实践要点 monitoring metrics).
    """
    N, k = cfg.n_experts, cfg.top_k
    counts = np.asarray(counts, dtype=np.float64)
    kept = np.asarray(kept, dtype=np.float64)
    f = counts / (k * T)
    P = normalised_affinity(s, cfg.score_fn).mean(axis=0) if T > 0 else np.zeros(N)
    aux_raw = N * float(np.sum(f * P))
    z = float(np.mean(lse ** 2)) if T > 0 else 0.0
    mean_c = counts.mean()
    cv = float(np.sqrt(np.mean((counts - mean_c) ** 2)) / mean_c) if mean_c > 0 else 0.0
    mean_k = kept.mean()
    cv_kept = float(np.sqrt(np.mean((kept - mean_k) ** 2)) / mean_k) if mean_k > 0 else 0.0
    return {"f": f, "P": P, "aux_raw": aux_raw, "aux": alpha * aux_raw, "z": z,
            "z_loss": z_coef * z, "cv": cv, "cv_kept": cv_kept,
            "dead": int(np.sum(counts == 0)), "dropped_slots": dropped_slots,
            "dropped_tokens": dropped_tokens,
            "bias_norm": 0.0 if bias is None else float(np.sqrt(np.sum(np.asarray(bias, np.float64) ** 2)))}


# ---------------------------------------------------------------------------
# 14. Aux-loss-free bias update
# ---------------------------------------------------------------------------
def bias_update(bias: np.ndarray, counts: np.ndarray, rate: float = 1e-3,
                clamp: Optional[float] = None) -> np.ndarray:
    """b[e] += rate * sign(mean(c) - c[e]) (sign(0) = 0), optional clamp to +-clamp.

    [Practice] BiasBalancedRouter.update_bias (overloaded experts pushed down,
    underloaded up, step 1e-3); [Compass] "负载均衡" describes the same direction.
    The batch is treated as one sequence.  The +-1e-2 clamp of [Practice] is an
    option that is off by default.
    """
    c = np.asarray(counts, dtype=np.float64)
    delta = c.mean() - c
    b = np.asarray(bias, dtype=np.float64) + rate * np.sign(delta)
    if clamp is not None and clamp > 0:
        b = np.clip(b, -clamp, clamp)
    return b


# ---------------------------------------------------------------------------
# Whole layer
# ---------------------------------------------------------------------------
ExpertWeights = Callable[[int], tuple]


def layer_forward(x: np.ndarray, w_gate: np.ndarray, cfg: OracleConfig,
                  expert_weights: ExpertWeights,
                  shared_weights: Optional[tuple] = None,
                  bias=None, logit_offset=None,
                  alpha: float = 0.0, z_coef: float = 0.0,
                  tokens: Optional[Sequence[int]] = None,
                  routing: Optional[dict] = None, expert_ffn=None) -> dict:
    """The layer forward in the pages' order: route, capacity/drop, permute,
    expert FFNs (+ shared), combine, statistics.

    expert_weights(e) returns (w1 [f, d], w3 [f, d], w2 [d, f]) for expert e, so
    large layers can widen one expert at a time.  `tokens`, when given, restricts
    the expert compute and combine to those tokens (routing, capacity and
    statistics still see every token).  `routing` lets a test feed a fixed
    routing decision (idx, w) instead of recomputing it.  `expert_ffn(x_rows, w1,
    w3, w2)` replaces the exact SwiGLU expert (e.g. swiglu_ffn_fp8).
    """
    T, d = x.shape
    ffn = swiglu_ffn if expert_ffn is None else expert_ffn
    r = route(x, w_gate, cfg, bias, logit_offset) if routing is None else routing
    C = capacity(cfg, T)
    p = permutation(r["idx"], cfg.n_experts, C)
    want = np.arange(T) if tokens is None else np.asarray(tokens)
    want_set = set(int(t) for t in want)
    y = np.zeros((len(want), d))
    if shared_weights is not None:
        y += ffn(np.asarray(x, np.float64)[want], *shared_weights)
    pos_in_want = {int(t): i for i, t in enumerate(want)}
    # gather, per expert, the rows (token, slot) that belong to wanted tokens
    for e in range(cfg.n_experts):
        lo, hi = p["offsets"][e], p["offsets"][e + 1]
        rows = [rr for rr in range(lo, hi) if int(p["token_of_row"][rr]) in want_set]
        if not rows:
            continue
        toks = p["token_of_row"][rows]
        ye = ffn(np.asarray(x, np.float64)[toks], *expert_weights(e))
        for i, rr in enumerate(rows):
            t = int(p["token_of_row"][rr])
            j = int(np.nonzero(p["row_of_slot"][t] == rr)[0][0])
            y[pos_in_want[t]] += r["w"][t, j] * ye[i]
    out = {"y": y, "tokens": want, "routing": r, "perm": p, "capacity": C}
    if "s" in r:
        out["stats"] = router_stats(p["counts"], p["kept"], r["s"], r["lse"], cfg, T,
                                    p["dropped_slots"], p["dropped_tokens"], alpha, z_coef, bias)
    return out


# ---------------------------------------------------------------------------
# Routing variants
# ---------------------------------------------------------------------------
def bias_update_ema(bias: np.ndarray, counts: np.ndarray, ema: np.ndarray, beta: float,
                    rate: float = 1e-3, clamp: Optional[float] = None) -> tuple:
    """Bias controller on an exponential moving average of the loads.

    [Landscape] (TL;DR, §2 and 实践要点) names an aux-loss-free "bias EMA" controller
    without a formula.  Reading: the smoothed load c~ <- beta c~ + (1 - beta) c
    replaces the current counts in the sign update of [Practice] update_bias,
    b_e += rate * sign(mean(c~) - c~_e).  beta = 0 is the plain update.
    Returns (new_bias, new_ema).
    """
    ema_new = beta * np.asarray(ema, np.float64) + (1.0 - beta) * np.asarray(counts, np.float64)
    delta = ema_new.mean() - ema_new
    b = np.asarray(bias, np.float64) + rate * np.sign(delta)
    if clamp is not None and clamp > 0:
        b = np.clip(b, -clamp, clamp)
    return b, ema_new


def sequence_load(idx: np.ndarray, seq_offsets: np.ndarray, n_experts: int) -> np.ndarray:
    """Per-expert load with every sequence weighted equally: sum_b c_be / len_b.

    [Practice] update_bias averages per-sequence counts "so long sequences do not
    dominate" and its long-context section suggests weighting by token counts.
    The printed form (mean over sequences of raw counts) equals the batch counts
    divided by the number of sequences, so its sign update is the batch update;
    reading for the variant: each sequence's counts are divided by its length
    (the share of that sequence's tokens routed to e), then summed over sequences
    (the 1/B factor does not change any sign).
    """
    load = np.zeros(n_experts)
    for b in range(len(seq_offsets) - 1):
        lo, hi = int(seq_offsets[b]), int(seq_offsets[b + 1])
        if hi > lo:
            load += np.bincount(idx[lo:hi].reshape(-1), minlength=n_experts) / float(hi - lo)
    return load


def bias_update_from_load(bias: np.ndarray, load: np.ndarray, rate: float = 1e-3,
                          clamp: Optional[float] = None) -> np.ndarray:
    """b_e += rate * sign(mean(load) - load_e) for a real-valued load."""
    load = np.asarray(load, np.float64)
    b = np.asarray(bias, np.float64) + rate * np.sign(load.mean() - load)
    if clamp is not None and clamp > 0:
        b = np.clip(b, -clamp, clamp)
    return b


def route_shared_sink(x, w_gate_ext, cfg: OracleConfig, bias=None, logit_offset=None) -> dict:
    """Router whose single shared expert joins the weight normalisation.

    [Taste] section 11 (shared-expert sink): the shared expert is normalised
    together with the selected routed experts, so it competes for mixture weight.
    Reading: w_gate_ext has N + 1 rows, row N scoring the shared expert; the
    affinity covers all N + 1 logits (softmax over N + 1, or independent
    sigmoids); top-k (and the group limit) choose among the N routed experts only;
    w_j = s_j / (sum_sel s + s_shared) and w_shared = s_shared / (same).
    """
    z = router_logits(x, w_gate_ext, None)
    if logit_offset is not None:
        z[:, :-1] = z[:, :-1] + np.asarray(logit_offset, np.float64)[None, :]
    s_all = affinity(z, cfg.score_fn)
    s, s_sh = s_all[:, :-1], s_all[:, -1]
    q = selection_scores(s, bias)
    mask, gmargin = eligible_mask(q, cfg)
    idx, emargin = select_topk(q, cfg.top_k, mask)
    sel = np.take_along_axis(s, idx, axis=1)
    den = sel.sum(axis=1) + s_sh
    return {"logits": z, "s": s, "s_shared": s_sh, "idx": idx, "w": sel / den[:, None],
            "w_shared": s_sh / den, "margin": np.minimum(emargin, gmargin), "lse": logsumexp(z)}


# ---------------------------------------------------------------------------
# Expert-choice routing
# ---------------------------------------------------------------------------
def expert_choice_capacity(n_experts: int, top_k: int, T: int, cf: float) -> int:
    """C = ceil(cf * k * T / N): each expert takes its share of the k T assignments
    ([Practice] "容量因子、token dropping": C = capacity_factor * k * T / n_experts),
    at most T."""
    return min(T, int(np.ceil((cf * top_k * T) / n_experts)))


def expert_choice(s: np.ndarray, C: int) -> dict:
    """Every expert takes the C tokens with the largest affinity.

    [Practice] "路由的数学形式" (last paragraphs) and [Landscape] §0: in expert-choice
    routing each expert picks its top-C tokens by its own capacity, so every expert
    is exactly full and no token is dropped by capacity (a token may be picked by no
    expert, or by several).  Readings: the affinity is the token-choice router's
    (softmax over experts); equal scores go to the lower token index; the gate weight
    of a picked pair is its affinity (no renormalisation); an expert's rows are its
    picked tokens in ascending token order.
    """
    T, N = s.shape
    row_of = np.full((N, T), -1, dtype=np.int64)
    token_of_row = np.zeros(N * C, dtype=np.int64)
    for e in range(N):
        order = np.argsort(-s[:, e], kind="stable")[:C]       # descending, lower token first on ties
        picked = np.sort(order)
        for i, t in enumerate(picked):
            row_of[e, t] = e * C + i
            token_of_row[e * C + i] = t
    picks = (row_of >= 0).sum(axis=0)
    return {"row_of": row_of, "token_of_row": token_of_row, "offsets": np.arange(N + 1) * C,
            "picks": picks, "unpicked": int((picks == 0).sum())}


def expert_choice_combine(y_rows: np.ndarray, row_of: np.ndarray, s: np.ndarray,
                          shared_out: Optional[np.ndarray]) -> np.ndarray:
    """y[t] = shared[t] + sum over experts e that picked t of s[t, e] * E_e(x[t])."""
    N, T = row_of.shape
    y = np.zeros((T, y_rows.shape[1])) if shared_out is None else np.array(shared_out, np.float64)
    for t in range(T):
        for e in range(N):
            r = row_of[e, t]
            if r >= 0:
                y[t] += s[t, e] * y_rows[r]
    return y


# ---------------------------------------------------------------------------
# FP8 expert compute (fine-grained block scaling)
# ---------------------------------------------------------------------------
E4M3_MAX = 448.0


def round_e4m3(v: np.ndarray) -> np.ndarray:
    """Round to the nearest FP8 E4M3 value (ties to even), saturating at +-448.

    E4M3 (OCP 8-bit floating point, "E4M3FN"): 4 exponent bits with bias 7 and 3
    mantissa bits; normal values (1 + m/8) 2^e for e in [-6, 8] (largest 1.75 * 2^8
    = 448), subnormals m 2^-9; no infinities.  Written from that definition.
    """
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    out = np.zeros_like(v)
    normal = a >= 2.0 ** -6
    e = np.floor(np.log2(np.where(normal, a, 1.0)))
    step = np.where(normal, 2.0 ** (e - 3), 2.0 ** -9)
    r = np.rint(a / step) * step                       # np.rint: round half to even
    out = np.sign(v) * np.minimum(r, E4M3_MAX)
    return out


def quantize_fp8_blocks(x: np.ndarray, block_rows: int, block_cols: int = 128) -> tuple:
    """Fine-grained FP8 quantisation: one scale per block_rows x block_cols block.

    [Taste] §2 (table of common taste vs frontier) lists FP8 / MXFP8 expert compute
    as a strong candidate and [Practice]
    "精度怎么定" says DeepSeek-V3 trains in FP8 with fine-grained precision assignment,
    without giving the scheme.  Reading (the DeepSeek-V3 one): 1 x 128 blocks for
    activations, 128 x 128 for weights; scale s = amax / 448 computed in fp32
    (s = 1 for an all-zero block), code q = E4M3(x / s) with x / s in fp32.
    Returns (dequantised codes q as float64, scales [ceil(rows/br), cols/bc]).
    """
    x32 = np.asarray(x, np.float32)
    R, Cc = x32.shape
    nbr, nbc = -(-R // block_rows), Cc // block_cols
    scales = np.zeros((nbr, nbc), np.float32)
    q = np.zeros((R, Cc), np.float64)
    for i in range(nbr):
        for j in range(nbc):
            blk = x32[i * block_rows:(i + 1) * block_rows, j * block_cols:(j + 1) * block_cols]
            amax = np.float32(np.max(np.abs(blk))) if blk.size else np.float32(0)
            s = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1.0)
            scales[i, j] = s
            q[i * block_rows:(i + 1) * block_rows, j * block_cols:(j + 1) * block_cols] = \
                round_e4m3((blk / s).astype(np.float32))
    return q, scales


def dequantize_fp8_blocks(q: np.ndarray, scales: np.ndarray, block_rows: int, block_cols: int = 128):
    s = np.repeat(np.repeat(np.asarray(scales, np.float64), block_rows, axis=0), block_cols, axis=1)
    return q * s[: q.shape[0], : q.shape[1]]


def swiglu_ffn_fp8(x_rows, w1, w3, w2, hidden_out: bool = False):
    """The SwiGLU expert with FP8 operands: x in 1 x 128 blocks, W in 128 x 128 blocks,
    fp64 accumulation of the dequantised products; the hidden h is quantised again
    (1 x 128 blocks) before the down projection."""
    xq, xs = quantize_fp8_blocks(x_rows, 1)
    xd = dequantize_fp8_blocks(xq, xs, 1)
    wd = [dequantize_fp8_blocks(*quantize_fp8_blocks(w, 128), 128) for w in (w1, w3, w2)]
    h = silu(xd @ wd[0].T) * (xd @ wd[1].T)
    hq, hs = quantize_fp8_blocks(h, 1)
    y = dequantize_fp8_blocks(hq, hs, 1) @ wd[2].T
    return (y, h) if hidden_out else y


# ---------------------------------------------------------------------------
# MXFP8 (OCP Microscaling) experts
# ---------------------------------------------------------------------------
MX_BLOCK = 32
E4M3_EMAX = 8          # exponent of E4M3's largest normal (448 = 1.75 * 2^8)


def quantize_mxfp8(x: np.ndarray, block: int = MX_BLOCK) -> tuple:
    """MXFP8 quantisation along each row: every `block` consecutive elements share
    one E8M0 scale 2^e.

    [Taste] §2 (table) names MXFP8 expert compute.  The format is the OCP
    Microscaling (MX) one: scale exponent e = floor(log2(amax)) - emax(E4M3), with
    emax(E4M3) = 8, clamped to the E8M0 range [-127, 127]; elements are
    E4M3(x / 2^e), saturating at 448 (a block's largest magnitude lands in
    [256, 512), so it may saturate).  An all-zero block takes e = -127.
    floor(log2(amax)) comes from frexp, which is exact.
    Returns (dequantisable codes as float64 values, exponents e [rows, cols/block] int).
    """
    x = np.asarray(x, np.float64)
    R, C = x.shape
    blocks = x.reshape(R, C // block, block)
    amax = np.max(np.abs(blocks), axis=2)
    _, ex = np.frexp(amax)                         # amax = m 2^ex, m in [0.5, 1)
    e = np.where(amax > 0, ex.astype(np.int64) - 1 - E4M3_EMAX, -127)
    e = np.clip(e, -127, 127)
    q = round_e4m3(blocks / (2.0 ** e)[:, :, None]).reshape(R, C)
    return q, e


def dequantize_mxfp8(q: np.ndarray, e: np.ndarray, block: int = MX_BLOCK) -> np.ndarray:
    return np.asarray(q, np.float64) * np.repeat(2.0 ** np.asarray(e, np.float64), block, axis=1)


def swiglu_ffn_mxfp8(x_rows, w1, w3, w2, hidden_out: bool = False):
    """The SwiGLU expert with MXFP8 operands: x, W1, W3 quantised along d and W2
    and h along d_ff (the contraction dimension, 1 x 32 blocks); fp64 products of
    the dequantised values."""
    xd = dequantize_mxfp8(*quantize_mxfp8(x_rows))
    w1d, w3d, w2d = (dequantize_mxfp8(*quantize_mxfp8(w)) for w in (w1, w3, w2))
    h = silu(xd @ w1d.T) * (xd @ w3d.T)
    y = dequantize_mxfp8(*quantize_mxfp8(h)) @ w2d.T
    return (y, h) if hidden_out else y


# ---------------------------------------------------------------------------
# NVFP4 experts
# ---------------------------------------------------------------------------
NVFP4_BLOCK = 16
E2M1_MAX = 6.0


def round_e2m1(v: np.ndarray) -> np.ndarray:
    """Round to the nearest FP4 E2M1 value (ties to even), saturating at +-6.

    E2M1: 1 sign bit, 2 exponent bits with bias 1, 1 mantissa bit; normal values
    (1 + m/2) 2^(e-1) for e in 1..3 (1, 1.5, 2, 3, 4, 6), subnormals m/2 (0, 0.5);
    no infinities or NaN.  The spacing is 0.5 below 2, then doubles per binade.
    Written from that definition.
    """
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    step = np.where(a >= 1.0, 2.0 ** (np.floor(np.log2(np.where(a >= 1.0, a, 1.0))) - 1.0), 0.5)
    r = np.rint(a / step) * step                       # np.rint: round half to even
    return np.sign(v) * np.minimum(r, E2M1_MAX)


def nvfp4_tensor_scale(x: np.ndarray) -> np.float32:
    """Per-tensor fp32 scale of the two-level NVFP4 scheme: amax / (6 * 448), so the
    block scales amax_b / (6 g) stay inside UE4M3's range; 1 for an all-zero tensor."""
    amax = np.float32(np.max(np.abs(np.asarray(x, np.float32)))) if np.size(x) else np.float32(0)
    return np.float32(amax / np.float32(E2M1_MAX * E4M3_MAX)) if amax > 0 else np.float32(1.0)


def quantize_nvfp4(x: np.ndarray, g: float = 1.0, block: int = NVFP4_BLOCK) -> tuple:
    """NVFP4 quantisation along each row with tensor scale g.

    [Taste] §2 (table) names NVFP4 expert compute without spelling it out.  Reading
    (NVIDIA's NVFP4): E2M1 elements, one unsigned E4M3 scale per 16 consecutive
    elements of the contraction dimension and one fp32 scale g per tensor.  In fp32,
    in this order: b = E4M3(amax_b / fp32(6 g)) (round to nearest even, saturating at
    448), s = fp32(b g), code = E2M1(fp32(x / s)); a block with b = 0 has all codes 0.
    Dequantised value: code * b * g.  Reading of the tensor scale: weights take
    nvfp4_tensor_scale (one per expert matrix); activations (x rows and the hidden h)
    take g = 1, their block maxima already lying in E4M3's normal range.
    Returns (codes as float64 values [R, C], block scales b [R, C / block] float64).
    """
    x32 = np.asarray(x, np.float32)
    R, C = x32.shape
    g = np.float32(g)
    blocks = x32.reshape(R, C // block, block)
    amax = np.max(np.abs(blocks), axis=2).astype(np.float32)
    denom = np.float32(np.float32(E2M1_MAX) * g)
    b = round_e4m3((amax / denom).astype(np.float32))
    s = (b.astype(np.float32) * g).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = (blocks / s[:, :, None]).astype(np.float32)
    q = np.where(b[:, :, None] > 0, round_e2m1(v), 0.0).reshape(R, C)
    return q, b


def dequantize_nvfp4(q: np.ndarray, b: np.ndarray, g: float = 1.0, block: int = NVFP4_BLOCK) -> np.ndarray:
    return np.asarray(q, np.float64) * np.repeat(np.asarray(b, np.float64), block, axis=1) * float(np.float32(g))


def swiglu_ffn_nvfp4(x_rows, w1, w3, w2, hidden_out: bool = False):
    """The SwiGLU expert with NVFP4 operands: x (g = 1), W1, W3 (each its own tensor
    scale) quantised along d, h (g = 1) and W2 along d_ff; fp64 products of the
    dequantised values."""
    xd = dequantize_nvfp4(*quantize_nvfp4(x_rows))

    def wq(w):
        g = nvfp4_tensor_scale(w)
        return dequantize_nvfp4(*quantize_nvfp4(w, g), g)

    w1d, w3d, w2d = wq(w1), wq(w3), wq(w2)
    h = silu(xd @ w1d.T) * (xd @ w3d.T)
    y = dequantize_nvfp4(*quantize_nvfp4(h)) @ w2d.T
    return (y, h) if hidden_out else y


# ---------------------------------------------------------------------------
# Expert parallelism: the exchange plan
# ---------------------------------------------------------------------------
def ep_plan(offsets_all: np.ndarray, rank: int) -> dict:
    """The bookkeeping of [Practice] "专家并行与 all-to-all" for rank `rank` of W:
    experts are sharded contiguously (rank of expert e = e // (N / W)); each rank
    knows every rank's per-expert kept counts (exchanged before the rows).

    offsets_all [W, N+1]: every rank's expert offsets (rows kept per expert are
    their differences).  Returns
      send[r]       rows this rank sends to rank r (its kept rows of r's experts),
      recv[s]       rows it receives from rank s,
      local_offsets exclusive scan over its experts of the rows received for each,
      regroup[q]    received row q -> local row, where received rows come source
                    rank major, then expert, then row (the all-to-all order) and
                    local rows come expert major, then source rank, then row.
    Written as explicit loops over (source, expert, row).
    """
    off = np.asarray(offsets_all, np.int64)
    W, N = off.shape[0], off.shape[1] - 1
    El = N // W
    kept = off[:, 1:] - off[:, :-1]
    mine = range(rank * El, (rank + 1) * El)
    send = [int(sum(kept[rank, r * El + j] for j in range(El))) for r in range(W)]
    recv = [int(sum(kept[s, e] for e in mine)) for s in range(W)]
    local_counts = [int(sum(kept[s, e] for s in range(W))) for e in mine]
    local_offsets = np.concatenate([[0], np.cumsum(local_counts)]).astype(np.int64)
    regroup = []
    for s in range(W):
        for j, e in enumerate(mine):
            before = sum(kept[s2, e] for s2 in range(s))
            for i in range(kept[s, e]):
                regroup.append(int(local_offsets[j] + before + i))
    return {"send": send, "recv": recv, "local_offsets": local_offsets, "regroup": np.array(regroup, np.int64)}
