"""One MoE FFN layer forward through the C ABI: buffers plus the call sequence.

This is orchestration only (allocation through torch, then route -> permute ->
grouped FFN (routed, shared) -> combine -> statistics -> bias update, all on one
stream); every step runs in the library's kernels.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _lib as L
from .synth import Workload, torch_dtype

CAP_MODES = {"dropless": L.CAP_DROPLESS, "ceil_cf_T_over_N": L.CAP_CEIL_CF_T_OVER_N,
             "floor_cf_k_T_over_N": L.CAP_CF_K_T_OVER_N_FLOOR}


def make_config(w: Workload, T: Optional[int] = None) -> L.MoeConfig:
    c = L.MoeConfig()
    c.T = w.T if T is None else T
    c.d_model, c.n_experts, c.top_k, c.d_ff = w.d, w.N, w.k, w.f
    c.score_fn = L.SCORE_SIGMOID if w.score == "sigmoid" else L.SCORE_SOFTMAX
    c.renorm = 1 if w.renorm else 0
    c.n_groups, c.topk_groups, c.group_score_topn = w.n_groups, w.topk_groups, w.group_topn
    c.capacity_mode = CAP_MODES[w.capacity]
    c.capacity_factor = w.cf
    c.x_dtype = L.DTYPE_F32 if w.dtype == "fp32" else L.DTYPE_BF16
    c.shared_sink = 1 if w.shared_sink else 0
    return c


class MoELayer:
    """Holds the weights and the per-call buffers of one layer for up to T tokens."""

    def __init__(self, w: Workload, weights: dict, device="cuda", update_bias: bool = True,
                 group=None, overlap_shared: Optional[bool] = None, gather_rows: bool = False,
                 fuse_shared: bool = True, split_shared: bool = True):
        """group: a torch.distributed process group when the layer runs as one of
        several data-parallel replicas; the router statistics are then those of the
        whole group's batch (each rank's sufficient statistics summed over the
        group) and the bias update uses the counts summed over the group, so all
        replicas keep the same selection bias."""
        lowp = w.fp8 or w.mxfp8 or w.nvfp4
        if w.expert_choice and lowp:
            raise ValueError("expert-choice routing runs bf16 or fp32 experts")
        if lowp and (w.dtype != "bf16" or w.d % 128 or w.f % 128 or w.f_shared % 128):
            raise ValueError("FP8 experts need bf16 inputs and d, d_ff multiples of 128")
        if w.nvfp4 and (w.d % 256 or w.f % 256 or (w.n_shared * w.f_shared) % 256):
            raise ValueError("NVFP4 experts need d and d_ff multiples of 256")
        self.w = w
        self.group = group
        # shared experts on a side stream, concurrently with route and permute (they do not
        # depend on the routing); joined before the combine.  With low-precision experts the
        # side stream also quantises x for them (the quantising scatter then writes only
        # the routed rows).  None: on for bf16 experts, off for low-precision ones, where
        # it measured no faster (the step is power-bound and the overlap adds no work saved)
        if overlap_shared is None:
            overlap_shared = not lowp
        self.overlap_shared = overlap_shared and w.n_shared > 0 and not w.expert_choice
        # gather_rows: bf16 experts read their rows straight from x (moe_grouped_ffn_gather),
        # so the permutation writes no expert-ordered copy of x (T k d elements less
        # memory); off by default: the first GEMM's row copies cost more time than the
        # copy they save
        self.gather_rows = (gather_rows and w.dtype == "bf16" and w.d % 64 == 0
                            and not (lowp or w.expert_choice))
        # fuse_shared: a bf16 shared expert of the routed experts' width runs as one more
        # group inside the routed grouped-FFN launches (moe_grouped_ffn_shared, or
        # moe_grouped_ffn_gather with the shared weights); its rows follow the routed rows
        # in h and y_perm
        self.fuse_shared = (fuse_shared and w.dtype == "bf16" and not (lowp or w.expert_choice)
                            and w.n_shared * w.f_shared == w.f and w.N < 512)
        if self.fuse_shared:
            self.overlap_shared = False
        # split_shared (with fuse_shared): the shared expert's first pass on a side stream,
        # concurrently with route and permute; its second pass inside the routed second
        # pass's launch (moe_grouped_ffn_gate_up / moe_grouped_ffn_down)
        self.split_shared = split_shared and self.fuse_shared and not self.gather_rows
        self.dev = torch.device(device)
        self.weights = weights
        self.update_bias = update_bias and weights.get("bias") is not None
        self.cfg = make_config(w)
        T, d, N, k = w.T, w.d, w.N, w.k
        dt = torch_dtype(w)
        z = lambda *s, dtype=torch.float32: torch.empty(s, dtype=dtype, device=self.dev)  # noqa: E731
        self.nblk = L.route_partials(self.cfg)
        self.topk_idx = z(T, k, dtype=torch.int32)
        self.topk_w = z(T, k)
        self.lse = z(T)
        self.p_partial = z(max(self.nblk, 1), N)
        self.margin = z(T)
        self.counts = z(N, dtype=torch.int32)
        self.offsets = z(N + 1, dtype=torch.int32)
        self.row_of_slot = z(T, k, dtype=torch.int32)
        self.token_of_row = z(max(T * k, 1), dtype=torch.int32)
        self.x_perm = None if self.gather_rows else z(max(T * k, 1), d, dtype=dt)
        self.n_dropped = z(2, dtype=torch.int32)
        self.ws = z(max(L.workspace_size(self.cfg), 16), dtype=torch.uint8)
        # the tensor-core router's exact bf16 split of W_g, written once (prepare_router)
        self.route_split = None
        if L.route_prepare_size(self.cfg) > 0 and not w.expert_choice:
            self.route_split = z(L.route_prepare_size(self.cfg), dtype=torch.uint8)
            self.prepare_router()
        self.fs = w.n_shared * w.f_shared
        extra = T if self.fuse_shared else 0         # the fused shared expert's rows
        self.h = z(max(T * k + extra, 1), w.f, dtype=dt)
        self.y_perm = z(max(T * k + extra, 1), d, dtype=dt)
        if self.fs > 0:
            self.shared_offsets = torch.tensor([0, T], dtype=torch.int32, device=self.dev)
            if self.fuse_shared:
                self.hs, self.ys = self.h[T * k:], self.y_perm[T * k:]
            else:
                self.hs = z(max(T, 1), self.fs, dtype=dt)
                self.ys = z(max(T, 1), d, dtype=dt)
        self.y = z(max(T, 1), d, dtype=dt)
        if lowp:
            self._init_fp8(z)
        self.stats = torch.zeros(L.STATS_BYTES, dtype=torch.uint8, device=self.dev)
        self.counts_global = z(N, dtype=torch.int32)
        self.stats_part = z(L.stats_partial_len(N), dtype=torch.float64)
        self.f_out = z(N)
        self.p_out = z(N)
        self.shared_w = z(max(T, 1)) if w.shared_sink else None
        if w.expert_choice:
            C = self.C = L.expert_choice_capacity(self.cfg)
            self.scores = z(N, max(T, 1))
            self.row_of = z(N, max(T, 1), dtype=torch.int32)
            self.token_of_row = z(max(N * C, 1), dtype=torch.int32)
            self.x_perm = z(max(N * C, 1), d, dtype=dt)
            self.h = z(max(N * C, 1), w.f, dtype=dt)
            self.y_perm = z(max(N * C, 1), d, dtype=dt)
            self.n_unpicked = z(1, dtype=torch.int32)

    def prepare_router(self, stream=None):
        """Split the router weight for the tensor-core router; call again after changing
        weights["w_gate"] in place."""
        if self.route_split is not None:
            L.moe_route_prepare(self.cfg, self.weights["w_gate"], self.route_split, stream)

    def route(self, x, stream=None):
        """moe_route on x into this layer's routing buffers."""
        W = self.weights
        if self.route_split is not None:
            wg, ws = None, self.route_split
        else:
            wg, ws = W["w_gate"], self.ws
        L.moe_route(self.cfg, x, wg, W.get("logit_offset"), W.get("bias"), self.topk_idx, self.topk_w, self.lse,
                    self.p_partial, self.margin, ws, stream, shared_w=self.shared_w)

    def _init_fp8(self, z):
        """Low-precision experts: quantise the weights once (fine-grained FP8: 128 x 128
        blocks with fp32 scales; MXFP8: 1 x 32 blocks along K with E8M0 scales; NVFP4:
        1 x 16 blocks along K with E4M3 scales and one fp32 scale per expert matrix) and
        hold code buffers for the permuted rows, the hidden rows and the shared experts'
        input in place of the bf16 ones."""
        w, W, T, d, N, k = self.w, self.weights, self.w.T, self.w.d, self.w.N, self.w.k
        u8 = torch.uint8
        mx, nv = w.mxfp8, w.nvfp4
        # scales of grouped (permuted) rows: tile atoms need one spare tile per group
        if nv:
            sfa = lambda rows, cols, groups=0: L.nv_scales(rows, cols, self.dev, groups)  # noqa: E731
        elif mx:
            sfa = lambda rows, cols, groups=0: L.mx_scales(rows, cols, self.dev, groups)  # noqa: E731
        else:
            sfa = lambda rows, cols, groups=0: z(rows, cols // 128)  # noqa: E731
        cw = (lambda cols: cols // 2) if nv else (lambda cols: cols)     # code bytes per row

        def quant_w(t):
            m = t.reshape(-1, t.shape[-1])
            q = z(m.shape[0], cw(m.shape[1]), dtype=u8)
            if nv:
                # one tensor scale per expert matrix (t is [experts, rows, cols] or one matrix)
                per = t.shape[-2]
                sc, g = L.nv_scales(m.shape[0], m.shape[1], self.dev), z(m.shape[0] // per)
                L.moe_quantize_nvfp4(m, q, sc, g, tensor_rows=per)
                return q, sc, g
            if mx:
                sc = L.mx_scales(m.shape[0], m.shape[1], self.dev)
                L.moe_quantize_mxfp8(m, q, sc)
            else:
                sc = z((m.shape[0] + 127) // 128, m.shape[1] // 128)
                L.moe_quantize_fp8(m, 128, q, sc)
            return q, sc

        self.wq = {name: quant_w(W[name]) for name in ("w1", "w3", "w2")}
        rows = max(T * k, 1)
        self.x_perm = self.h = None
        self.xq_perm, self.xs_perm = z(rows, cw(d), dtype=u8), sfa(rows, d, N)
        self.hq, self.hsc = z(rows, cw(w.f), dtype=u8), sfa(rows, w.f, N)
        if self.fs > 0:
            self.wq.update({name: quant_w(W[name]) for name in ("ws1", "ws3", "ws2")})
            self.xq, self.xs = z(max(T, 1), cw(d), dtype=u8), sfa(max(T, 1), d)
            self.hq_sh, self.hsc_sh = z(max(T, 1), cw(self.fs), dtype=u8), sfa(max(T, 1), self.fs)
            self.hs = None

    def _ffn_fp8(self, c, xq, xs, rows, offsets, G, names, f, hq, hsc, y, s):
        w1, w3, w2 = (self.wq[n] for n in names)
        if self.w.nvfp4:
            L.moe_grouped_ffn_nvfp4(c, xq, xs, rows, offsets, G, *w1, *w3, *w2, f, hq, hsc, y, s)
            return
        fn = L.moe_grouped_ffn_mxfp8 if self.w.mxfp8 else L.moe_grouped_ffn_fp8
        fn(c, xq, xs, rows, offsets, G, *w1, *w3, *w2, f, hq, hsc, y, s)

    # the launches of one layer forward; `x` is [T, d] on the device.  `marks`, if
    # given, is a list of 7 CUDA events recorded between the stages (route, permute,
    # routed FFN, shared FFN, combine, statistics + bias update).
    def forward(self, x: torch.Tensor, stream=None, marks=None, out=None) -> torch.Tensor:
        W, c, T = self.weights, self.cfg, self.w.T
        y = self.y if out is None else out
        s = stream if stream is not None else torch.cuda.current_stream(self.dev)
        rec = (lambda i: marks[i].record(s)) if marks is not None else (lambda i: None)
        if self.w.expert_choice:
            return self._forward_ec(x, s, rec, y)
        lowp = self.w.fp8 or self.w.mxfp8 or self.w.nvfp4
        rec(0)
        join = None
        side_work = self.overlap_shared or self.split_shared
        if side_work:
            fork = torch.cuda.Event()
            fork.record(s)
        self.route(x, s)
        if side_work:
            if not hasattr(self, "_side"):
                self._side = torch.cuda.Stream(self.dev)
            side = self._side
            side.wait_event(fork)
            with torch.cuda.stream(side):
                if lowp:
                    if self.w.nvfp4:
                        L.moe_quantize_nvfp4(x, self.xq, self.xs, stream=side)
                    elif self.w.mxfp8:
                        L.moe_quantize_mxfp8(x, self.xq, self.xs, side)
                    else:
                        L.moe_quantize_fp8(x, 1, self.xq, self.xs, side)
                    self._ffn_fp8(c, self.xq, self.xs, T, self.shared_offsets, 1, ("ws1", "ws3", "ws2"), self.fs,
                                  self.hq_sh, self.hsc_sh, self.ys, side)
                elif self.split_shared:
                    L.moe_grouped_ffn_gate_up(c, x, T, self.shared_offsets, 1, W["ws1"], W["ws3"], self.fs, self.hs,
                                              side)
                else:
                    L.moe_grouped_ffn(c, x, T, self.shared_offsets, 1, W["ws1"], W["ws3"], W["ws2"], self.fs,
                                      self.hs, self.ys, side)
            join = torch.cuda.Event()
            join.record(side)
        rec(1)
        fp8 = lowp
        tok = self.fs > 0 and not self.overlap_shared     # the shared experts' input, from the scatter
        L.moe_permute(c, x, self.topk_idx, self.counts, self.offsets, self.row_of_slot,
                      self.token_of_row, self.x_perm, self.n_dropped, self.ws, s)
        if self.w.nvfp4:
            L.moe_permute_nvfp4(c, x, self.topk_idx, self.row_of_slot, self.offsets, self.xq_perm, self.xs_perm,
                                self.xq if tok else None, self.xs if tok else None, s)
        elif self.w.mxfp8:
            L.moe_permute_mxfp8(c, x, self.topk_idx, self.row_of_slot, self.offsets, self.xq_perm, self.xs_perm,
                                self.xq if tok else None, self.xs if tok else None, s)
        elif fp8:
            L.moe_permute_fp8(c, x, self.row_of_slot, self.xq_perm, self.xs_perm,
                              self.xq if tok else None, self.xs if tok else None, s)
        rec(2)
        if fp8:
            self._ffn_fp8(c, self.xq_perm, self.xs_perm, T * self.w.k, self.offsets, self.w.N,
                          ("w1", "w3", "w2"), self.w.f, self.hq, self.hsc, self.y_perm, s)
        elif self.gather_rows:
            sw = (W["ws1"], W["ws3"], W["ws2"]) if self.fuse_shared else (None, None, None)
            L.moe_grouped_ffn_gather(c, x, T, self.token_of_row, T * self.w.k, self.offsets, self.w.N, W["w1"],
                                     W["w3"], W["w2"], self.w.f, self.h, self.y_perm, s, *sw)
        elif self.split_shared:
            L.moe_grouped_ffn_gate_up(c, self.x_perm, T * self.w.k, self.offsets, self.w.N, W["w1"], W["w3"],
                                      self.w.f, self.h, s)
            s.wait_event(join)                 # the shared expert's first pass
            join = None
            L.moe_grouped_ffn_down(c, self.h, T * self.w.k, self.offsets, self.w.N, W["w2"], self.w.f, self.y_perm,
                                   T, W["ws2"], s)
        elif self.fuse_shared:
            L.moe_grouped_ffn_shared(c, self.x_perm, T * self.w.k, self.offsets, self.w.N, W["w1"], W["w3"],
                                     W["w2"], self.w.f, self.h, self.y_perm, x, T, W["ws1"], W["ws3"], W["ws2"], s)
        else:
            L.moe_grouped_ffn(c, self.x_perm, T * self.w.k, self.offsets, self.w.N, W["w1"], W["w3"],
                              W["w2"], self.w.f, self.h, self.y_perm, s)
        rec(3)
        shared = None
        if self.fs > 0:
            if join is not None:
                s.wait_event(join)
            elif self.fuse_shared:
                pass                   # computed with the routed experts
            elif fp8:
                self._ffn_fp8(c, self.xq, self.xs, T, self.shared_offsets, 1, ("ws1", "ws3", "ws2"),
                              self.fs, self.hq_sh, self.hsc_sh, self.ys, s)
            else:
                L.moe_grouped_ffn(c, x, T, self.shared_offsets, 1, W["ws1"], W["ws3"], W["ws2"],
                                  self.fs, self.hs, self.ys, s)
            shared = self.ys
        rec(4)
        L.moe_combine(c, self.y_perm, self.row_of_slot, self.topk_w, shared, y, s,
                      shared_w=self.shared_w)
        rec(5)
        counts = self.counts
        if self.group is None:
            L.moe_router_stats(c, self.counts, self.offsets, self.p_partial, self.lse, self.n_dropped,
                               W.get("bias"), self.w.alpha, self.w.z_coef, self.stats, self.f_out,
                               self.p_out, s, margin=self.margin)
        else:
            # statistics of the whole group's batch: sum the sufficient statistics
            from .replicas import all_reduce_sum
            L.moe_router_stats_partial(c, self.counts, self.offsets, self.p_partial, self.lse, self.n_dropped,
                                       self.stats_part, margin=self.margin, stream=s)
            with torch.cuda.stream(s):
                all_reduce_sum(self.stats_part, self.group)
            L.moe_router_stats_finalize(c, self.stats_part, W.get("bias"), self.w.alpha, self.w.z_coef,
                                        self.stats, self.f_out, self.p_out, self.counts_global, s)
            counts = self.counts_global
        if self.update_bias:
            L.moe_bias_update(c, counts, W["bias"], self.w.bias_rate, 0.0, s)
        rec(6)
        return y

    def _forward_ec(self, x, s, rec, y):
        """Expert-choice routing: scores -> per-expert top-C -> grouped FFN -> combine."""
        W, c, w = self.weights, self.cfg, self.w
        rec(0)
        L.moe_route_scores(c, x, W["w_gate"], W.get("logit_offset"), self.scores, self.lse,
                           self.p_partial, self.ws, s)
        rec(1)
        L.moe_expert_choice(c, x, self.scores, self.C, self.row_of, self.token_of_row, self.offsets,
                            self.x_perm, self.n_unpicked, s)
        rec(2)
        L.moe_grouped_ffn(c, self.x_perm, w.N * self.C, self.offsets, w.N, W["w1"], W["w3"], W["w2"],
                          w.f, self.h, self.y_perm, s)
        rec(3)
        shared = None
        if self.fs > 0:
            L.moe_grouped_ffn(c, x, w.T, self.shared_offsets, 1, W["ws1"], W["ws3"], W["ws2"], self.fs,
                              self.hs, self.ys, s)
            shared = self.ys
        rec(4)
        L.moe_combine_ec(c, self.y_perm, self.row_of, self.scores, shared, y, self.n_unpicked, s)
        rec(5)
        rec(6)
        return y

    def capture(self, x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.cuda.CUDAGraph:
        """Record one whole forward on the fixed input buffer `x` into a CUDA graph
        (after one eager forward on the capture stream, which sets the kernels' launch
        attributes); `replay()` then reruns every launch of the step, the bias update
        included, without host launch overhead.  Not for the replica mode (its counts
        all-reduce is a collective)."""
        if self.group is not None:
            raise ValueError("capture is for a single-process layer")
        s = torch.cuda.Stream(self.dev)
        s.wait_stream(torch.cuda.current_stream(self.dev))
        with torch.cuda.stream(s):
            self.forward(x, s, out=out)
        torch.cuda.current_stream(self.dev).wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            self.forward(x, s, out=out)
        self._graph = g
        return g

    def replay(self):
        self._graph.replay()

    def forward_host(self, x_host_steps, y_host_steps, stream=None):
        """Layer forwards on host data: for each step, copy its [T, d] input from
        pinned host memory, run the layer, copy the result back into the matching
        pinned host output.  Uploads, compute and downloads run on three streams
        with two device input/output buffers, so step i+1's upload and step i-1's
        download overlap step i's compute; every step still moves its own input
        and result.  Returns after enqueueing; synchronise before reading outputs."""
        comp = stream if stream is not None else torch.cuda.current_stream(self.dev)
        if not hasattr(self, "_pipe"):
            T, d = self.w.T, self.w.d
            dt = self.y.dtype
            self._pipe = {
                "x": [torch.empty(max(T, 1), d, dtype=dt, device=self.dev) for _ in range(2)],
                "y": [torch.empty(max(T, 1), d, dtype=dt, device=self.dev) for _ in range(2)],
                "up": torch.cuda.Stream(self.dev), "down": torch.cuda.Stream(self.dev),
                "x_ready": [torch.cuda.Event() for _ in range(2)],
                "x_free": [torch.cuda.Event() for _ in range(2)],
                "y_ready": [torch.cuda.Event() for _ in range(2)],
                "y_free": [torch.cuda.Event() for _ in range(2)],
            }
        P = self._pipe
        up, down = P["up"], P["down"]
        # the first uploads must not overtake work already queued on the compute stream
        up.wait_stream(comp)
        down.wait_stream(comp)
        for i, (xh, yh) in enumerate(zip(x_host_steps, y_host_steps)):
            b = i % 2
            up.wait_event(P["x_free"][b])
            with torch.cuda.stream(up):
                P["x"][b].copy_(xh, non_blocking=True)
                P["x_ready"][b].record(up)
            comp.wait_event(P["x_ready"][b])
            comp.wait_event(P["y_free"][b])
            self.forward(P["x"][b], comp, out=P["y"][b])
            P["x_free"][b].record(comp)
            P["y_ready"][b].record(comp)
            down.wait_event(P["y_ready"][b])
            with torch.cuda.stream(down):
                yh.copy_(P["y"][b][: yh.shape[0]], non_blocking=True)
                P["y_free"][b].record(down)
        comp.wait_stream(down)

    def kernel_launches(self) -> int:
        """Number of the library's kernels one forward launches."""
        if self.w.expert_choice:       # scores (+ split), select, gather, FFN (2), combine
            n = 1 + 2 + 2 + 1 + (1 if self.w.dtype == "bf16" and self.w.N <= 256 else 0)
            return n + (2 if self.fs > 0 else 0)
        n = 1 + 4 + 2 + 1 + 1          # route, permute (4), routed FFN (2), combine, stats
        if self.group is not None:
            n += 1                     # statistics in two launches around the all-reduce
        # FP8: the permutation's bf16 gather is replaced by the quantising scatter;
        # the router weight's split is written once, outside the forward
        if self.gather_rows:
            n -= 1                     # no row gather: the grouped FFN reads x itself
        if self.fs > 0 and not self.fuse_shared:
            n += 2
        if self.split_shared:
            n += 1                     # the shared expert's first pass in a launch of its own
        if self.update_bias:
            n += 1
        return n

    def stats_dict(self) -> dict:
        return L.stats_from_tensor(self.stats)
