"""Benchmark of the MoE FFN layer forward on the DeepSeek-V3-shaped workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one whole layer forward (route, permute, routed + shared grouped SwiGLU
FFN, combine, router statistics, bias update) over T = 16384 tokens of d = 7168,
256 routed experts top-8 (d_ff 2048), 1 shared expert, sigmoid + selection bias,
8 groups keep 4, dropless; seeded synthetic inputs resident in HBM.  Inputs are
larger than L2 (x = 235 MB, expert weights 22.5 GB), so no L2 flush is needed.
With N > 1 (torchrun) every rank runs its own 16384 tokens against replicated
experts (weak scaling, no data-path collective); the time is the max over ranks.

`--impl reference` times the plain fp64 CPU oracle on a bounded token sample of
the same workload on the host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

WORKLOAD = "deepseek_v3"
METRIC = "MoE layer fwd tokens/s"
UNIT = "tokens/s"

# DRAM bytes (read + write) of one routed grouped-FFN call (its kernels' launches of
# one forward) from an ncu capture of those kernels alone with the one-pass metrics
# dram__bytes_read.sum, dram__bytes_write.sum, gpu__time_duration.sum; valid only
# while every listed kernel source is the one that was profiled (sha1), else null.
NCU_TRAFFIC = {
    # reduced case (T = 4096, 64 experts, shared expert in launches of its own), scaled to
    # the full layer: routed bytes x 4, the shared expert's rows x 4 plus its 88 MB of
    # weights once; profiles/ffn_deepseek_v3_reduced.md
    "deepseek_v3": ({"ffn_tc.cu": "2c6f53fa57720d650812402c7e1362c7f837f184"}, 28.7e9),
    # reduced case (T = 4096, 64 experts), routed passes only, x 4;
    # profiles/ffn_mx_traffic_deepseek_v3_mxfp8_reduced.md
    "deepseek_v3_mxfp8": ({"ffn_mx.cu": "2e97d1168131256a9632d796c2ebb5de99a384a6"}, 15.04e9),
}


# The shared expert's first pass (its W1/W3 once, its rows x 4 from the same reduced capture):
# DRAM bytes that leave the grouped-FFN stage when that pass runs on a side stream.
SPLIT_SHARED_GATE_UP_BYTES = {"deepseek_v3": 0.58e9}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def _sha1(path):
    return hashlib.sha1(open(path, "rb").read()).hexdigest()


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region
    (all GPUs are sampled; lines are kept for the device's UUID)."""
    Q = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        rows = [[x.strip() for x in ln.split(",")] for ln in self.lines]
        rows = [r for r in rows if len(r) >= 9]
        mine = [r for r in rows if self.uuid and self.uuid in r[0]]
        if not mine and len({r[0] for r in rows}) == 1:
            mine = rows
        sm, smax, power, reasons = [], None, [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in mine:
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
                power.append(float(r[3]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "power_w_median": statistics.median(power) if power else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def _device_uuid(dev):
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


def _oracle_cfg(O, w):
    cap = {"dropless": O.CAP_DROPLESS, "ceil_cf_T_over_N": O.CAP_CEIL_CF_T_OVER_N,
           "floor_cf_k_T_over_N": O.CAP_CF_K_T_OVER_N_FLOOR}[w.capacity]
    return O.OracleConfig(n_experts=w.N, top_k=w.k, score_fn=O.SIGMOID if w.score == "sigmoid" else O.SOFTMAX,
                          renorm=w.renorm, n_groups=w.n_groups, topk_groups=w.topk_groups,
                          group_score_topn=w.group_topn, capacity_mode=cap, capacity_factor=w.cf)


# ---------------------------------------------------------------------------- reference arm
def run_reference(args, rank):
    """The fp64 CPU oracle on a bounded sample of the workload, host cores."""
    if rank != 0:
        return 0
    from oracle import moe_oracle as O
    from sparse_mixture_experts_21_b200.synth import WORKLOADS, make_inputs

    w = WORKLOADS[args.workload]
    sample = args.ref_tokens
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(w, dev)
    cfg = _oracle_cfg(O, w)
    f64 = lambda t: None if t is None else t.detach().cpu().to(torch.float64).numpy()  # noqa: E731
    wg, bias, off = f64(inp["w_gate"]), f64(inp["bias"]), f64(inp["logit_offset"])
    shared = (f64(inp["ws1"]), f64(inp["ws3"]), f64(inp["ws2"])) if w.n_shared else None
    ffn = (O.swiglu_ffn_fp8 if w.fp8 else O.swiglu_ffn_mxfp8 if w.mxfp8 else
           O.swiglu_ffn_nvfp4 if w.nvfp4 else None)

    def experts(e):
        return f64(inp["w1"][e]), f64(inp["w3"][e]), f64(inp["w2"][e])

    def step(i):
        t0 = (i * sample) % w.T
        x = f64(inp["x"][t0:t0 + sample])
        O.layer_forward(x, wg, cfg, experts, shared, bias=bias, logit_offset=off, alpha=w.alpha,
                        z_coef=w.z_coef, expert_ffn=ffn)

    for i in range(args.warmup):
        step(i)
    t = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = (time.perf_counter() - t) / max(args.steps, 1)
    value = sample / dt
    cores = len(os.sched_getaffinity(0))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": dict(workload_config(w, args.gpus), sample_tokens_per_step=sample),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{sample} tokens per step of the {w.name} workload "
                                       f"(full routing, experts, shared expert, combine, stats)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, world: int = 1) -> dict:
    """The workload's description, the same in both arms' lines."""
    return {"workload": w.name, "T": w.T, "d_model": w.d, "experts": w.N, "top_k": w.k, "d_ff": w.f,
            "shared_experts": w.n_shared,
            "score": w.score + ("+bias" if w.bias_std > 0 else ""),
            "groups": f"{w.n_groups} keep {w.topk_groups}" if w.n_groups > 1 else "none",
            "routing": "expert-choice" if w.expert_choice else "token-choice top-k",
            "capacity": w.capacity, "parallelism": f"replicas x{world}",
            "experts_precision": ("E4M3, 1x128 / 128x128 block scales" if w.fp8 else
                                  "MXFP8: E4M3, E8M0 scale per 32 along K" if w.mxfp8 else
                                  "NVFP4: E2M1, E4M3 scale per 16 along K, fp32 per expert matrix"
                                  if w.nvfp4 else "fp32" if w.dtype == "fp32" else "bf16")}


# ---------------------------------------------------------------------------- our arm
def cpu_baseline(inp, w, seconds_target=20.0, chunk=4, max_tokens=64, threads=None):
    """Oracle timed on a bounded sample (the first tokens of the same workload, `chunk`
    tokens per oracle call, until `seconds_target` or `max_tokens`; a workload smaller
    than the sample is run again from its first token).  threads: cap on the BLAS
    threads (None: every host core)."""
    from threadpoolctl import threadpool_limits

    from oracle import moe_oracle as O
    cfg = _oracle_cfg(O, w)
    f64 = lambda t: None if t is None else t.detach().cpu().to(torch.float64).numpy()  # noqa: E731
    wg, bias, off = f64(inp["w_gate"]), f64(inp["bias"]), f64(inp["logit_offset"])
    shared = (f64(inp["ws1"]), f64(inp["ws3"]), f64(inp["ws2"])) if w.n_shared else None
    ffn = (O.swiglu_ffn_fp8 if w.fp8 else O.swiglu_ffn_mxfp8 if w.mxfp8 else
           O.swiglu_ffn_nvfp4 if w.nvfp4 else None)

    def experts(e):
        return f64(inp["w1"][e]), f64(inp["w3"][e]), f64(inp["w2"][e])

    cores = len(os.sched_getaffinity(0)) if threads is None else threads
    done, t0 = 0, time.perf_counter()
    with threadpool_limits(limits=cores):
        while True:
            t0_ = done % w.T                       # wraps around small workloads
            x = f64(inp["x"][t0_:t0_ + chunk])
            O.layer_forward(x, wg, cfg, experts, shared, bias=bias, logit_offset=off, alpha=w.alpha,
                            z_coef=w.z_coef, expert_ffn=ffn)
            done += chunk
            el = time.perf_counter() - t0
            if el > seconds_target or done >= max_tokens:
                break
    return {"value": done / el, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{done} tokens of the {w.name} workload from its first, {chunk} per oracle call "
                      f"(routing, experts, shared expert, combine, stats), {el:.1f} s"}


def run_cpu_baselines(args):
    """The oracle on every workload of the task (host cores; also one core for the
    three smaller ones): one JSON line per (workload, cores).  Inputs are drawn on the
    GPU with the workload's seed, so they are the bytes the GPU path sees."""
    from sparse_mixture_experts_21_b200.synth import WORKLOADS, make_inputs
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    plan = [("tiny_top2_fp32", 256, 256 * 1000, (None, 1)), ("mixtral_8x7b", 8, 64, (None, 1)),
            ("deepseekmoe_16b", 32, 256, (None, 1)), ("deepseek_v3", 4, 64, (None,)),
            ("switch_skewed", 64, 1024, (None,))]
    for name, chunk, max_tokens, cores in plan:
        w = WORKLOADS[name]
        inp = make_inputs(w, dev)
        for c in cores:
            r = cpu_baseline(inp, w, seconds_target=args.cpu_seconds, chunk=chunk, max_tokens=max_tokens,
                             threads=c)
            print(json.dumps({"workload": name, **r}), flush=True)
        del inp
        if dev == "cuda":
            torch.cuda.empty_cache()
    return 0


def run_ep(args, w, world, rank, local, dev, pg):
    """Expert parallelism: every rank routes its own T tokens, holds N / W experts, and
    exchanges rows with the others (all-to-all dispatch and return, in rounds bounded
    by the receive buffer).  Weak scaling: T tokens per rank."""
    from sparse_mixture_experts_21_b200 import _lib as L
    from sparse_mixture_experts_21_b200.ep import EPMoELayer, TorchDistExchange
    from sparse_mixture_experts_21_b200.replicas import max_over_ranks
    from sparse_mixture_experts_21_b200.synth import make_inputs

    if pg is None:
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29531")
        dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist
    inp = make_inputs(w, dev, seed=0)                       # router and experts: the same on every rank
    x = make_inputs(w, dev, seed=100 + rank, experts=False)["x"]  # this rank's tokens
    peer = args.ep_exchange == "peer"
    lay = EPMoELayer(w, inp, rank, world, dev, exchange=TorchDistExchange(), recv_factor=args.recv_factor,
                     peer=peer, device_plan=peer and args.ep_plan == "device")
    for name in ("w1", "w3", "w2"):                         # only this rank's experts stay resident
        inp[name] = None
    torch.cuda.empty_cache()
    stream = torch.cuda.current_stream(dev)

    def barrier():
        pg.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        lay.forward(x)
    barrier()
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    marks = [[ev() for _ in range(4)] for _ in range(args.steps)]
    rounds = []
    with ClockSampler(_device_uuid(local)) as clk:
        barrier()
        start, end = ev(), ev()
        start.record(stream)
        for i in range(args.steps):
            lay.forward(x, stream, marks[i])
            rounds.append(len(lay.plans) if world > 1 and not lay.device_plan else 1)
        end.record(stream)
        barrier()
    ms = max_over_ranks(start.elapsed_time(end) / args.steps, dev)
    assert L.moe_device_status() == L.MOE_OK
    stage = lambda a, b: statistics.mean(marks[i][a].elapsed_time(marks[i][b]) for i in range(args.steps))  # noqa: E731
    t_route_perm, t_expert, t_finish = stage(0, 1), stage(1, 2), stage(2, 3)
    t_expert_max = max_over_ranks(t_expert, dev)
    # rows this rank's experts computed in the last step, and their FLOPs
    R_local = lay.rows_received()
    flops_local = 6.0 * R_local * w.d * w.f
    peaks = _peaks()
    tflops = flops_local / (t_expert * 1e-3) / 1e12
    st = lay.base.stats_dict()

    # end to end: each step copies its tokens from pinned host memory and its output back
    xh = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    xh.copy_(x)
    yh = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    xd = torch.empty_like(x)
    barrier()
    s0, s1 = ev(), ev()
    s0.record(stream)
    for _ in range(args.steps):
        xd.copy_(xh, non_blocking=True)
        y = lay.forward(xd)
        yh.copy_(y[: w.T], non_blocking=True)
    s1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(s0.elapsed_time(s1) / args.steps, dev)
    if rank == 0:
        line = {
            "metric": METRIC, "value": world * w.T / (ms * 1e-3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "T_per_rank": w.T, "d_model": w.d, "experts": w.N, "top_k": w.k,
                       "d_ff": w.f, "shared_experts": w.n_shared, "parallelism": f"ep{world}",
                       "experts_per_rank": w.N // world,
                       "recv_factor": None if lay.device_plan else args.recv_factor,
                       "exchange": args.ep_exchange if world > 1 else "none (one rank)",
                       "plan": ("device" if lay.device_plan else "host") if world > 1 else "none (one rank)",
                       "rounds_per_step": max(rounds) if rounds else 1,
                       "l2": "inputs larger than L2 (x 235 MB per rank, local expert weights "
                             f"{3 * (w.N // world) * w.d * w.f * 2 / 1e9:.1f} GB); no flush"},
            "roofline": {"kernel": "exchange + local grouped SwiGLU FFN (rank 0)", "bound": "tensor",
                         "achieved": tflops, "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                         "frac": tflops / peaks["bf16_tflops_sustained"], "traffic": None,
                         "peak_source": peaks["source"] + " sustained bf16"},
            "stages_ms": {"route_permute": t_route_perm, "exchange_and_experts": t_expert,
                          "exchange_and_experts_max_over_ranks": t_expert_max, "shared_combine_stats": t_finish},
            "near_ties": {"count": st["near_ties"], "tokens": st["T"], "threshold": L.NEAR_TIE},
            "gpu_launches": lay.kernel_launches() * args.steps,
            "clocks": clk.summary(),
            "e2e": {"value": world * w.T / (e2e_ms * 1e-3), "unit": UNIT,
                    "h2d_bytes_per_step": xh.numel() * xh.element_size(),
                    "d2h_bytes_per_step": yh.numel() * yh.element_size(), "ms_per_step": e2e_ms,
                    "api": "EPMoELayer.forward (pinned host in/out per step)"},
            "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)
    torch.cuda.synchronize(dev)
    pg.barrier()                      # every rank is done with every other rank's buffers
    lay.close()
    pg.barrier()
    pg.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-tokens", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-baselines", action="store_true",
                    help="time the oracle on every workload (host cores, and one core for the smaller ones)")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay measurement")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="workload name from synth.WORKLOADS (default: the DeepSeek-V3-shaped layer)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="reduced token count (profiling of a small case only)")
    ap.add_argument("--experts", type=int, default=None,
                    help="reduced routed-expert count (profiling of a small case only)")
    ap.add_argument("--parallel", default="replicas", choices=["replicas", "ep"],
                    help="replicas: every rank holds every expert; ep: expert parallelism (N / W experts per "
                         "rank, all-to-all dispatch and return)")
    ap.add_argument("--no-overlap-shared", action="store_true",
                    help="run the shared experts on the main stream after the routed experts (default: bf16 "
                         "shared experts that are not fused run on a side stream, concurrently with route and "
                         "permute; low-precision ones on the main stream)")
    ap.add_argument("--no-fuse-shared", action="store_true",
                    help="run the shared expert in launches of its own instead of as one more group of the "
                         "routed grouped-FFN launches")
    ap.add_argument("--no-split-shared", action="store_true",
                    help="bf16, shared expert fused: run both of its passes inside the routed launches (default: "
                         "its first pass on a side stream during route and permute, its second pass inside the "
                         "routed down launch)")
    ap.add_argument("--gather-rows", action="store_true",
                    help="bf16: the grouped FFN gathers its rows from x (cp.async) instead of reading the "
                         "expert-ordered copy that the permutation writes")
    ap.add_argument("--recv-factor", type=float, default=1.0,
                    help="ep: receive buffer rows as a multiple of T * k (rounds bound it)")
    ap.add_argument("--ep-plan", default="device", choices=["device", "host"],
                    help="ep with the peer exchange: device -- receive buffers sized for every row a rank can "
                         "receive, one round, no host synchronisation; host -- rounds bounded by --recv-factor, "
                         "planned on the host")
    ap.add_argument("--ep-exchange", default="peer", choices=["peer", "nccl"],
                    help="ep: peer -- the library's kernels store rows into the other ranks' receive buffers "
                         "and read the results back over NVLink peer memory (CUDA IPC mappings); nccl -- "
                         "batched NCCL point-to-point transfers")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)
    if args.cpu_baselines:
        return run_cpu_baselines(args) if rank == 0 else 0

    from sparse_mixture_experts_21_b200 import _lib as L
    from sparse_mixture_experts_21_b200.layer import MoELayer
    from sparse_mixture_experts_21_b200.synth import WORKLOADS, make_inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    L.load()
    w = WORKLOADS[args.workload]
    if args.tokens or args.experts:
        from dataclasses import replace
        w = replace(w, name=w.name + "_reduced", T=args.tokens or w.T, N=args.experts or w.N)
    if args.parallel == "ep":
        return run_ep(args, w, world, rank, local, dev, pg)
    inp = make_inputs(w, dev, seed=rank)
    lay = MoELayer(w, inp, dev, group=None if pg is None else pg.group.WORLD, overlap_shared=False if args.no_overlap_shared else None,
                   gather_rows=args.gather_rows, fuse_shared=not args.no_fuse_shared,
                   split_shared=not args.no_split_shared)
    x = inp["x"]
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        lay.forward(x)
    barrier()

    # timed region: K whole-layer steps, events between the stages for per-stage times
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    marks = [[ev() for _ in range(7)] for _ in range(args.steps)]
    with ClockSampler(_device_uuid(local)) as clk:
        barrier()
        start, end = ev(), ev()
        start.record(stream)
        for i in range(args.steps):
            lay.forward(x, stream, marks[i])
        end.record(stream)
        barrier()
    ms_local = start.elapsed_time(end) / args.steps
    ms = ms_local
    if pg is not None:
        from sparse_mixture_experts_21_b200.replicas import max_over_ranks
        ms = max_over_ranks(ms_local, dev)
    assert L.moe_device_status() == L.MOE_OK
    st = lay.stats_dict()          # the last timed step's router statistics

    stage = lambda a, b: statistics.mean(marks[i][a].elapsed_time(marks[i][b]) for i in range(args.steps))  # noqa: E731
    t_route, t_perm, t_ffn, t_shared, t_comb, t_stats = (stage(0, 1), stage(1, 2), stage(2, 3),
                                                         stage(3, 4), stage(4, 5), stage(5, 6))
    # With the shared expert's first pass on a side stream, the route and permute stages
    # share the GPU with it, so their HBM figures come from a few more steps in the fused
    # form (both shared passes inside the routed launches), after the timed region.
    hbm_stages = "the timed steps"
    t_route_h, t_perm_h, t_comb_h = t_route, t_perm, t_comb
    if lay.split_shared:
        n_h = min(args.steps, 10)
        lay.split_shared = False
        marks_h = [[ev() for _ in range(7)] for _ in range(n_h)]
        for _ in range(2):
            lay.forward(x)
        for i in range(n_h):
            lay.forward(x, stream, marks_h[i])
        barrier()
        lay.split_shared = True
        stage_h = lambda a, b: statistics.mean(marks_h[i][a].elapsed_time(marks_h[i][b]) for i in range(n_h))  # noqa: E731
        t_route_h, t_perm_h, t_comb_h = stage_h(0, 1), stage_h(1, 2), stage_h(4, 5)
        hbm_stages = (f"{n_h} steps after the timed region with the shared expert fused into the routed "
                      "launches (in the timed steps its first pass shares the GPU with route and permute)")
    R = int(lay.offsets[-1].item())
    eb = 4 if w.dtype == "fp32" else 2
    T, d, N, k, f = w.T, w.d, w.N, w.k, w.f
    flops_routed = 6.0 * R * d * f
    flops_shared = 6.0 * T * d * lay.fs
    flops_router = 2.0 * T * d * N
    bytes_route = T * d * eb + 4 * N * d + 8 * T * k
    bytes_perm = T * d * eb + R * d * eb + 12 * T * k
    if lay.gather_rows:        # no row gather: index maps only (the grouped FFN reads x itself)
        bytes_perm = 12 * T * k
    bytes_comb = R * d * eb + 2 * T * d * eb + 8 * T * k
    lowp = w.fp8 or w.mxfp8 or w.nvfp4
    if lowp:                   # bf16 x read once; codes + scales written per row (+ token order)
        per_elem = 0.5 + 1 / 16 if w.nvfp4 else 1 + (4 / 128 if w.fp8 else 1 / 32)
        bytes_perm = T * d * eb + (R + (T if lay.fs else 0)) * d * per_elem + 12 * T * k
    if w.expert_choice:        # scores [N, T] written; rows gathered per row; combine reads the maps
        bytes_route = T * d * eb + 4 * N * d + 4 * N * T
        bytes_perm = 2 * R * d * eb + 12 * N * T
        bytes_comb = R * d * eb + 2 * T * d * eb + 8 * N * T
    peaks = _peaks()
    # E4M3 operands: the measured bf16 peak times the nominal fp8 / bf16 ratio (4.5 / 2.25);
    # E2M1 operands: times the nominal fp4 / bf16 ratio (9 / 2.25)
    ratio = 4.0 if w.nvfp4 else 2.0 if lowp else 1.0
    ffn_peak = peaks["bf16_tflops_sustained"] * ratio
    ffn_peak_src = peaks["source"] + (" sustained bf16 x 4 (nominal fp4/bf16 ratio)" if w.nvfp4 else
                                      " sustained bf16 x 2 (nominal fp8/bf16 ratio)" if lowp else " sustained bf16")
    ffn_bound = "tensor"
    if w.dtype == "fp32":
        # fp32 experts run on the FMA pipes: 148 SMs x 128 lanes x 2 FLOP x 1.965 GHz
        ffn_peak, ffn_bound = 148 * 128 * 2 * 1.965e9 / 1e12, "alu"
        ffn_peak_src = "derived: 148 SMs x 128 fp32 lanes x 2 FLOP x 1965 MHz"
    # with the shared expert fused into the routed launches, the stage does both
    # (split: the shared expert's first pass runs on a side stream before the stage, its
    # second pass -- a third of its FLOPs -- inside the stage's down launch)
    flops_ffn = flops_routed + (flops_shared / 3.0 if lay.split_shared else flops_shared if lay.fuse_shared
                                else 0.0)
    tflops_ffn = flops_ffn / (t_ffn * 1e-3) / 1e12
    traffic = None
    if w.name in NCU_TRAFFIC:
        srcs, nbytes = NCU_TRAFFIC[w.name]
        if all(_sha1(os.path.join(ROOT, "sparse_mixture_experts_21_b200", "csrc", f)) == h for f, h in srcs.items()):
            traffic = nbytes
            if lay.split_shared and w.name in SPLIT_SHARED_GATE_UP_BYTES:
                # the stage no longer holds the shared expert's first pass
                traffic -= SPLIT_SHARED_GATE_UP_BYTES[w.name]

    # the same step replayed from a CUDA graph (one capture, K replays): launch overhead out
    graph = None
    if pg is None and not args.no_graph:
        lay.capture(x)
        barrier()
        g0, g1 = ev(), ev()
        g0.record(stream)
        for _ in range(args.steps):
            lay.replay()
        g1.record(stream)
        barrier()
        gms = g0.elapsed_time(g1) / args.steps
        graph = {"value": T / (gms * 1e-3), "unit": UNIT, "ms_per_step": gms}
        assert L.moe_device_status() == L.MOE_OK

    # end to end through the public API: every step copies its input from pinned host
    # memory and its result back to pinned host memory (MoELayer.forward_host, which
    # overlaps one step's copies with the neighbouring steps' compute)
    e2e = None
    if not args.no_e2e:
        xh = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
        xh.copy_(x)
        yh = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
        lay.forward_host([xh] * 2, [yh] * 2, stream)
        barrier()
        s0, s1 = ev(), ev()
        s0.record(stream)
        lay.forward_host([xh] * args.steps, [yh] * args.steps, stream)
        s1.record(stream)
        barrier()
        e2e_ms = s0.elapsed_time(s1) / args.steps
        if pg is not None:
            from sparse_mixture_experts_21_b200.replicas import max_over_ranks
            e2e_ms = max_over_ranks(e2e_ms, dev)
        e2e = {"value": world * T / (e2e_ms * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": xh.numel() * xh.element_size(),
               "d2h_bytes_per_step": yh.numel() * yh.element_size(), "ms_per_step": e2e_ms,
               "api": "MoELayer.forward_host (pinned host in/out per step, copies overlapped)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(inp, w)

    if rank == 0:
        line = {
            "metric": METRIC, "value": world * T / (ms * 1e-3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": ("nvfp4-e2m1 experts, fp32 router" if w.nvfp4 else
                                                              "mxfp8-e4m3 experts, fp32 router" if w.mxfp8 else
                                                              "fp8-e4m3 experts, fp32 router" if w.fp8 else
                                                              "fp32" if w.dtype == "fp32" else "bf16"),
            "data": "synthetic",
            "config": dict(workload_config(w, world), rows_R=R,
                           expert_rows=("read from x by the first grouped GEMM (cp.async)" if lay.gather_rows
                                        else "expert-ordered copy of x written by the permutation"),
                           l2=(f"inputs larger than L2 (x {T * d * eb / 1e6:.0f} MB, expert weights "
                               f"{3 * N * d * f * (0.5 if w.nvfp4 else 1 if lowp else eb) / 1e9:.1f} GB); "
                               "no flush")),
            "tflops": (flops_routed + flops_shared + flops_router) / (ms * 1e-3) / 1e12,
            "roofline": {"kernel": ("grouped SwiGLU FFN, routed gate/up pass + routed and shared down pass"
                                    if lay.split_shared else
                                    "grouped SwiGLU FFN, routed + shared experts in one tile list (gate/up + "
                                    "down passes)" if lay.fuse_shared else
                                    "grouped SwiGLU FFN, routed experts (gate/up + down passes)"),
                         "bound": ffn_bound, "achieved": tflops_ffn,
                         "peak": ffn_peak, "unit": "TFLOP/s",
                         "frac": tflops_ffn / ffn_peak, "traffic": traffic,
                         "peak_source": ffn_peak_src},
            "stages_ms": {"route": t_route, "permute": t_perm, "routed_ffn": t_ffn,
                          "shared_ffn": t_shared, "combine": t_comb, "stats_bias": t_stats},
            "hbm": {"route_gbs": bytes_route / (t_route_h * 1e-3) / 1e9,
                    "permute_gbs": bytes_perm / (t_perm_h * 1e-3) / 1e9,
                    "combine_gbs": bytes_comb / (t_comb_h * 1e-3) / 1e9,
                    "peak_gbs": peaks["hbm_gbs"], "stages": hbm_stages},
            # on a side stream the shared experts overlap route, permute and the routed
            # experts; the main stream's "shared_ffn" stage is then only the join
            "shared_ffn_tflops": (None if (lay.overlap_shared or lay.fuse_shared or lay.fs == 0)
                                  else flops_shared / (t_shared * 1e-3) / 1e12),
            "shared_experts": ("first pass on a side stream during route and permute, second pass in the "
                               "routed down launch" if lay.split_shared else
                               "fused into the routed grouped-FFN launches" if lay.fuse_shared else
                               "side stream (overlapped)" if lay.overlap_shared else
                               "main stream" if lay.fs > 0 else "none"),
            "router_tflops_fp32": flops_router / (t_route_h * 1e-3) / 1e12,
            "router_stats": {"aux": st["aux"], "z_loss": st["z_loss"], "cv": st["cv"], "dead": st["dead"],
                             "dropped_slots": st["dropped_slots"], "dropped_tokens": st["dropped_tokens"]},
            "near_ties": {"count": st["near_ties"], "tokens": st["T"], "threshold": L.NEAR_TIE,
                          "frac": st["near_ties"] / max(st["T"], 1)},
            "gpu_launches": lay.kernel_launches() * args.steps,
            "clocks": clk.summary(),
            "e2e": e2e,
            "cuda_graph": graph,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
