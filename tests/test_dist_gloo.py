"""Multi-rank host logic of the replica mode, on CPU with two gloo ranks.

Each rank routes its own tokens; the per-expert counts are summed over ranks
before the bias update, so every replica applies the same update, equal to the
update a single process would apply to the concatenated batch.  The step time
reported is the maximum over ranks.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import moe_oracle as O
from sparse_mixture_experts_21_b200.replicas import all_reduce_counts, max_over_ranks
from sparse_mixture_experts_21_b200.synth import random_routing

N, K, T_PER_RANK, WORLD = 32, 4, 300, 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        idx = random_routing(T_PER_RANK, N, K, "cpu", seed=100 + rank, hot=rank)
        counts = torch.bincount(idx.reshape(-1).long(), minlength=N).to(torch.int32)
        glob = torch.empty_like(counts)
        all_reduce_counts(counts, glob)
        bias = O.bias_update(np.zeros(N), glob.numpy(), rate=1e-3)
        worst = max_over_ranks(1.5 + rank, "cpu")
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), idx=idx.numpy(), counts=counts.numpy(),
                 glob=glob.numpy(), bias=bias, worst=worst)
    finally:
        dist.destroy_process_group()


def test_replicas_share_counts_and_bias(tmp_path):
    mp.start_processes(_worker, args=(_free_port(), str(tmp_path)), nprocs=WORLD, join=True,
                       start_method="spawn")
    r = [np.load(tmp_path / f"r{i}.npz") for i in range(WORLD)]
    all_idx = np.concatenate([x["idx"] for x in r])
    want = np.bincount(all_idx.reshape(-1), minlength=N)
    for x in r:
        assert np.array_equal(x["glob"], want)              # global counts on every rank
        assert float(x["worst"]) == 2.5                     # max over ranks
    assert not np.array_equal(r[0]["counts"], r[1]["counts"])
    assert np.array_equal(r[0]["bias"], r[1]["bias"])       # replicas stay identical
    single = O.bias_update(np.zeros(N), want, rate=1e-3)
    assert np.array_equal(r[0]["bias"], single)             # same as one process on all tokens


# ----------------------------------------------------------------------------- expert parallelism
EP_N, EP_WORLD, EP_D = 8, 2, 16


def _ep_worker(rank, port, out_dir):
    """Rank `rank` exchanges rows with TorchDistExchange on CPU (gloo): the offsets
    all-gather, the dispatch all-to-all in the plan's split sizes, and the return
    all-to-all.  Each row carries (source rank, source row) so the receiver can
    check where it came from."""
    from sparse_mixture_experts_21_b200.ep import TorchDistExchange
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=EP_WORLD)
    try:
        ex = TorchDistExchange()
        rng = np.random.default_rng(300 + rank)
        kept = rng.integers(0, 6, size=EP_N)
        kept[rank * 3] = 0                                    # an empty expert on each rank
        offsets = torch.tensor(np.concatenate([[0], np.cumsum(kept)]), dtype=torch.int32)
        offsets_all = ex.all_gather(offsets)
        plan = O.ep_plan(offsets_all.numpy(), rank)
        R = int(kept.sum())
        send = torch.zeros(R, EP_D)
        send[:, 0] = rank
        send[:, 1] = torch.arange(R, dtype=torch.float32)
        recv = torch.full((sum(plan["recv"]), EP_D), -1.0)
        ex.all_to_all(recv, send, plan["recv"], plan["send"])
        # the "expert" here: add 1000 to every received row, then send it back
        back = torch.empty_like(send)
        ex.all_to_all(back, recv + 1000.0, plan["send"], plan["recv"])
        np.savez(os.path.join(out_dir, f"ep{rank}.npz"), offsets_all=offsets_all.numpy(), recv=recv.numpy(),
                 back=back.numpy(), send=send.numpy())
    finally:
        dist.destroy_process_group()


def test_ep_exchange_two_ranks(tmp_path):
    mp.start_processes(_ep_worker, args=(_free_port(), str(tmp_path)), nprocs=EP_WORLD, join=True,
                       start_method="spawn")
    r = [np.load(tmp_path / f"ep{i}.npz") for i in range(EP_WORLD)]
    assert np.array_equal(r[0]["offsets_all"], r[1]["offsets_all"])
    off = r[0]["offsets_all"]
    El = EP_N // EP_WORLD
    for rank in range(EP_WORLD):
        recv = r[rank]["recv"]
        # received rows: source-rank major, each source's rows of this rank's experts in order
        q = 0
        for s in range(EP_WORLD):
            lo, hi = off[s, rank * El], off[s, (rank + 1) * El]
            n = hi - lo
            assert np.all(recv[q:q + n, 0] == s)
            assert np.array_equal(recv[q:q + n, 1], np.arange(lo, hi))
            q += n
        assert q == len(recv)
        # every row comes home, in place, transformed once
        assert np.array_equal(r[rank]["back"], r[rank]["send"] + 1000.0)


# ----------------------------------------------------------------------------- global router statistics
ST_N, ST_K, ST_T, ST_D = 16, 3, 120, 12


def _stats_vector(x, wg, cfg):
    """The sufficient-statistics layout of moe_router_stats_partial, from the oracle:
    c_e, kept_e, sum_t s-hat_te, then sum_t lse^2, T, dropped slots, dropped tokens,
    near-ties (margin < 1e-4)."""
    r = O.route(x, wg, cfg)
    p = O.permutation(r["idx"], cfg.n_experts, O.capacity(cfg, x.shape[0]))
    shat = O.normalised_affinity(r["s"], cfg.score_fn)
    return np.concatenate([p["counts"], p["kept"], shat.sum(axis=0),
                           [np.sum(r["lse"] ** 2), x.shape[0], p["dropped_slots"], p["dropped_tokens"],
                            np.sum(r["margin"] < 1e-4)]])


def _stats_worker(rank, port, out_dir):
    from sparse_mixture_experts_21_b200.replicas import all_reduce_sum
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        rng = np.random.default_rng(500)
        wg = rng.normal(size=(ST_N, ST_D))
        x = np.random.default_rng(600 + rank).normal(size=(ST_T, ST_D))
        cfg = O.OracleConfig(ST_N, ST_K, score_fn=O.SIGMOID)
        v = torch.tensor(_stats_vector(x, wg, cfg), dtype=torch.float64)
        all_reduce_sum(v)
        np.savez(os.path.join(out_dir, f"st{rank}.npz"), v=v.numpy(), x=x, wg=wg)
    finally:
        dist.destroy_process_group()


def test_global_stats_vector_is_the_concatenated_batch(tmp_path):
    """Every rank's sufficient statistics summed over two gloo ranks equal those of the
    concatenated batch (dropless, so routing is per token), and the statistics
    computed from them are the oracle's statistics of the concatenated batch."""
    mp.start_processes(_stats_worker, args=(_free_port(), str(tmp_path)), nprocs=WORLD, join=True,
                       start_method="spawn")
    r = [np.load(tmp_path / f"st{i}.npz") for i in range(WORLD)]
    assert np.array_equal(r[0]["v"], r[1]["v"])
    cfg = O.OracleConfig(ST_N, ST_K, score_fn=O.SIGMOID)
    x_all = np.concatenate([r[i]["x"] for i in range(WORLD)])
    want = _stats_vector(x_all, r[0]["wg"], cfg)
    n = ST_N
    assert np.array_equal(r[0]["v"][:2 * n], want[:2 * n])                       # integer counts exact
    assert np.allclose(r[0]["v"][2 * n:], want[2 * n:], rtol=1e-13, atol=0)
    # aux from the summed vector = the oracle's aux on the concatenated batch
    v, T = r[0]["v"], WORLD * ST_T
    aux_raw = n * np.sum((v[:n] / (ST_K * T)) * (v[2 * n:3 * n] / T))
    out = O.layer_forward(x_all, r[0]["wg"], cfg, lambda e: (np.zeros((2, ST_D)), np.zeros((2, ST_D)),
                                                             np.zeros((ST_D, 2))))
    assert abs(aux_raw - out["stats"]["aux_raw"]) < 1e-12
    assert abs(v[3 * n] / T - out["stats"]["z"]) < 1e-12
