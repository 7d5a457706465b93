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
        ex.all_to_all(list(torch.split(recv, plan["recv"])), list(torch.split(send, plan["send"])))
        # the "expert" here: add 1000 to every received row, then send it back
        back = torch.empty_like(send)
        ex.all_to_all(list(torch.split(back, plan["send"])), list(torch.split(recv + 1000.0, plan["recv"])))
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


def _peer_worker(rank, port, out_dir):
    """The peer exchange's host side on CPU (gloo): every rank exports a handle of its
    buffer, the handles are all-gathered, each rank imports the others' and keeps its
    own address; barrier() is a collective every rank passes; release_peer closes
    exactly the imported addresses.  The library's CUDA IPC calls are replaced by
    fakes that encode (rank, address) in the handle."""
    import sparse_mixture_experts_21_b200.ep as E
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=EP_WORLD)
    try:
        closed = []
        L = E.L
        L.moe_peer_export = lambda t: (np.array([rank, t.data_ptr()], dtype=np.int64).tobytes()
                                       + bytes(L.PEER_HANDLE_BYTES - 16))
        L.moe_peer_import = lambda h: int(np.frombuffer(h[:16], dtype=np.int64)[1]) + 7   # "mapped" address
        L.moe_peer_close = lambda a: closed.append(a)
        ex = E.TorchDistExchange(device="cpu")
        buf = torch.zeros(4, 8)
        addrs = ex.peer_addresses(buf)
        ex.barrier()
        ex.barrier()
        others = [a for r, a in enumerate(addrs) if r != rank]
        for a in others:
            ex.release_peer(a)
        np.savez(os.path.join(out_dir, f"peer{rank}.npz"), addrs=np.array(addrs, dtype=np.int64),
                 own=buf.data_ptr(), closed=np.array(closed, dtype=np.int64), flag=ex._flag.numpy())
    finally:
        dist.destroy_process_group()


def test_peer_handles_exchange_two_ranks(tmp_path):
    mp.start_processes(_peer_worker, args=(_free_port(), str(tmp_path)), nprocs=EP_WORLD, join=True,
                       start_method="spawn")
    r = [np.load(tmp_path / f"peer{i}.npz") for i in range(EP_WORLD)]
    for rank in range(EP_WORLD):
        addrs = r[rank]["addrs"]
        assert addrs[rank] == int(r[rank]["own"])                    # its own buffer, not imported
        for o in range(EP_WORLD):
            if o != rank:
                assert addrs[o] == int(r[o]["own"]) + 7              # the other rank's handle, imported
        assert sorted(r[rank]["closed"].tolist()) == sorted(int(addrs[o]) for o in range(EP_WORLD) if o != rank)
        assert int(r[rank]["flag"][0]) == 0                          # the barrier's all-reduce of zeros


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


# ----------------------------------------------------------------------------- bounded EP exchange rounds
def test_round_plan_invariants():
    """Every (source, expert) piece goes to exactly one round, no destination receives
    more than the capacity in a round, and both ends agree on every split size."""
    from sparse_mixture_experts_21_b200.ep import plan_rounds, round_plans
    rng = np.random.default_rng(77)
    for W, N, cap in [(2, 8, 40), (4, 16, 60), (4, 16, 10 ** 6), (8, 64, 150)]:
        kept = rng.integers(0, 30, size=(W, N))
        kept[:, 3] = 0
        kept[0, N - 1] = cap                              # one piece exactly at the capacity
        off = np.concatenate([np.zeros((W, 1), np.int64), np.cumsum(kept, axis=1)], axis=1)
        round_of, R = plan_rounds(kept, W, cap)
        plans = [round_plans(off, r, W, cap) for r in range(W)]
        El = N // W
        for r in range(R):
            for d in range(W):
                assert sum(plans[d][r].recv_count) <= cap
                for s in range(W):
                    assert plans[s][r].send_count[d] == plans[d][r].recv_count[s]
                    # the slice a source sends is its rows of exactly this round's pieces
                    es = [e for e in range(d * El, (d + 1) * El) if round_of[s, e] == r]
                    assert plans[s][r].send_count[d] == sum(kept[s, e] for e in es)
        for s in range(W):                                # every row leaves once over the rounds
            assert sum(sum(p.send_count) for p in plans[s]) == kept[s].sum()
        if cap >= kept.sum():
            assert R == 1


def test_device_plan_capacity_always_fits_one_round():
    """The device-side plan's receive buffer, W * T * min(k, N / W) rows, holds every row a
    rank can receive: random routings, skewed ones and the worst case (every token of every
    rank picks k experts of one rank) all plan into a single round."""
    from sparse_mixture_experts_21_b200.ep import plan_rounds
    from sparse_mixture_experts_21_b200.synth import random_routing
    rng = np.random.default_rng(5)
    for W, N, k, T in [(2, 8, 2, 50), (4, 16, 4, 64), (4, 8, 6, 40), (8, 64, 8, 30)]:
        El = N // W
        cap = W * T * min(k, El)
        cases = []
        for seed in range(3):
            idx = [random_routing(T, N, k, "cpu", seed=100 * seed + r, hot=(r if seed == 1 else None)).numpy()
                   for r in range(W)]
            cases.append(np.stack([np.bincount(i.reshape(-1), minlength=N) for i in idx]))
        # worst case: every token of every rank picks experts of rank 0 only (min(k, El) of them)
        worst = np.zeros((W, N), np.int64)
        worst[:, :min(k, El)] = T
        cases.append(worst)
        for kept in cases:
            recv = [int(kept[:, d * El:(d + 1) * El].sum()) for d in range(W)]
            assert max(recv) <= cap
            _, R = plan_rounds(kept, W, cap)
            assert R == 1
        assert int(worst[:, :El].sum()) == cap                 # the bound is reached


EPR_N, EPR_WORLD, EPR_D, EPR_CAP = 8, 2, 4, 7


def _ep_round_worker(rank, port, out_dir):
    """The round protocol of EPMoELayer on CPU (gloo): per round the dispatch all-to-all
    of the plan's slices, an "expert" (+1000, then regroup by local expert is not needed
    for this check), and the return all-to-all into the source's slots."""
    from sparse_mixture_experts_21_b200.ep import TorchDistExchange, round_plans
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=EPR_WORLD)
    try:
        ex = TorchDistExchange()
        rng = np.random.default_rng(900 + rank)
        kept = rng.integers(0, 6, size=EPR_N)
        offsets = torch.tensor(np.concatenate([[0], np.cumsum(kept)]), dtype=torch.int32)
        off_all = ex.all_gather(offsets).numpy()
        plans = round_plans(off_all, rank, EPR_WORLD, EPR_CAP)
        R = int(kept.sum())
        x = torch.zeros(R, EPR_D)
        x[:, 0] = rank
        x[:, 1] = torch.arange(R, dtype=torch.float32)
        y = torch.full((R, EPR_D), -1.0)
        got = []
        for p in plans:
            recv = torch.full((sum(p.recv_count), EPR_D), -5.0)
            q = np.concatenate([[0], np.cumsum(p.recv_count)])
            ex.all_to_all([recv[q[s]:q[s + 1]] for s in range(EPR_WORLD)],
                          [x[a:a + n] for a, n in zip(p.send_start, p.send_count)])
            got.append(recv.clone())
            out = recv + 1000.0
            ex.all_to_all([y[a:a + n] for a, n in zip(p.send_start, p.send_count)],
                          [out[q[s]:q[s + 1]] for s in range(EPR_WORLD)])
        np.savez(os.path.join(out_dir, f"epr{rank}.npz"), x=x.numpy(), y=y.numpy(), n_rounds=len(plans),
                 recv=np.concatenate(got) if got else np.zeros((0, EPR_D)), off_all=off_all)
    finally:
        dist.destroy_process_group()


def test_ep_round_exchange_two_ranks(tmp_path):
    """With a receive capacity of 7 rows the exchange takes several rounds; every row
    reaches the rank that owns its expert exactly once and comes back, transformed
    once, to its own slot."""
    mp.start_processes(_ep_round_worker, args=(_free_port(), str(tmp_path)), nprocs=EPR_WORLD, join=True,
                       start_method="spawn")
    r = [np.load(tmp_path / f"epr{i}.npz") for i in range(EPR_WORLD)]
    assert int(r[0]["n_rounds"]) == int(r[1]["n_rounds"]) > 1
    off = r[0]["off_all"]
    El = EPR_N // EPR_WORLD
    for rank in range(EPR_WORLD):
        assert np.array_equal(r[rank]["y"], r[rank]["x"] + 1000.0)
        recv = r[rank]["recv"]
        want = sorted((s, i) for s in range(EPR_WORLD) for i in range(off[s, rank * El], off[s, (rank + 1) * El]))
        assert sorted(zip(recv[:, 0].astype(int).tolist(), recv[:, 1].astype(int).tolist())) == want
