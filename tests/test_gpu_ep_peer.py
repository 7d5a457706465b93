"""The expert-parallel exchange over peer memory, on one GPU.

* moe_ep_peer_plan against the oracle's expert-parallel plan: a row's address is
  its rank's receive buffer + (its local row in the oracle's regroup) * row bytes,
  for all rows and for the pieces of one round; rows past the receive buffer get no
  address and record an invalid argument;
* W ranks emulated in one process (their receive buffers are buffers of this GPU,
  so the kernels' peer addresses are plain device addresses): the dispatch fills
  every receive buffer in local-expert order, the collect returns every row, and the
  row-address combine equals moe_combine bit for bit;
* EPMoELayer(peer=True).forward for W ranks run as threads on one GPU: every rank's
  output equals the single-rank layer's on its tokens, in one round and in several, and
  with the plan kept on the device (receive buffers for every row a rank can receive);
  rank 0's output is also within the bf16 bar of the oracle's layer forward;
* two processes on one GPU with the library's CUDA IPC mapping: each imports the
  other's receive buffers and runs the peer forward, the barriers on the host (gloo
  plus a device synchronisation), so no kernel of one process waits for the other's.
"""
from __future__ import annotations

import os
import socket
import threading
from dataclasses import replace

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_21_b200 import _lib as L
from sparse_mixture_experts_21_b200.ep import EPMoELayer, round_plans
from sparse_mixture_experts_21_b200.layer import MoELayer
from sparse_mixture_experts_21_b200.synth import WORKLOADS, make_inputs, random_routing
from tests.parity_util import NEAR_TIE, TOL_BF16, expert_weights_fn, f64, i64, oracle_cfg, rel_err, shared_weights

pytestmark = pytest.mark.gpu

ROW_BYTES = 512


def _case(T=300):
    return replace(WORKLOADS["deepseek_v3"], name="v3_ep_small", T=T, d=256, N=32, k=4, f=256, n_groups=4,
                   topk_groups=2, n_shared=1, f_shared=256)


def _offsets(kept):
    W = kept.shape[0]
    return np.concatenate([np.zeros((W, 1), np.int64), np.cumsum(kept, axis=1)], axis=1).astype(np.int32)


def _want_addresses(off_round, off_own, rank, bases, row_bytes):
    """Row i of `rank` (expert e, piece in the round) -> bases[d] + local row * row_bytes,
    the local row taken from the oracle's regroup of d's arrival order (source major)."""
    W, N = off_round.shape[0], off_round.shape[1] - 1
    El = N // W
    kept_r = (off_round[:, 1:] - off_round[:, :-1]).astype(np.int64)
    want = np.zeros(int(off_own[N]), np.uint64)
    for d in range(W):
        p = O.ep_plan(off_round, d)
        q0 = int(sum(p["recv"][:rank]))                 # d's arrivals from sources before rank
        q = q0
        for e in range(d * El, (d + 1) * El):
            for i in range(int(kept_r[rank, e])):
                want[int(off_own[e]) + i] = np.uint64(bases[d] + int(p["regroup"][q]) * row_bytes)
                q += 1
    return want


@pytest.mark.parametrize("W,N", [(1, 8), (2, 32), (4, 16), (8, 256)])
def test_ep_peer_plan_matches_oracle(W, N):
    rng = np.random.default_rng(7 * W + N)
    kept = rng.integers(0, 40, size=(W, N))
    kept[:, 1] = 0
    off = _offsets(kept)
    bases = [(d + 1) << 36 for d in range(W)]          # addresses only: the plan never dereferences them
    peer_rows = torch.tensor(bases, dtype=torch.int64, device="cuda")
    off_d = torch.tensor(off, device="cuda")
    for rank in range(W):
        rows = int(off[rank, N])
        addr = torch.full((rows + 3,), -1, dtype=torch.int64, device="cuda")
        L.moe_ep_peer_plan(off_d, off_d[rank], W, rank, peer_rows, ROW_BYTES, 1 << 20, addr)
        torch.cuda.synchronize()
        got = addr.cpu().numpy().view(np.uint64)
        assert np.array_equal(got[:rows], _want_addresses(off, off[rank], rank, bases, ROW_BYTES)), rank
        assert np.all(addr[rows:].cpu().numpy() == -1)            # past this rank's rows: untouched
    assert L.moe_device_status() == L.MOE_OK


def test_ep_peer_plan_one_round_of_several():
    W, N, T, k = 4, 16, 200, 4
    idx = [random_routing(T, N, k, "cpu", seed=40 + r, hot=r).numpy() for r in range(W)]
    kept = np.stack([np.bincount(i.reshape(-1), minlength=N) for i in idx])
    off = _offsets(kept)
    cap = int(kept.max()) + 20                          # small: several rounds
    bases = [(d + 3) << 36 for d in range(W)]
    peer_rows = torch.tensor(bases, dtype=torch.int64, device="cuda")
    plans = [round_plans(off, rank, W, cap) for rank in range(W)]
    R = len(plans[0])
    assert R > 1
    own = torch.tensor(off, device="cuda")
    for r in range(R):
        off_r = plans[0][r].offsets_all                  # every rank derives the same round offsets
        off_rd = torch.tensor(off_r, device="cuda")
        for rank in range(W):
            rows = int(off[rank, N])
            addr = torch.full((rows,), -1, dtype=torch.int64, device="cuda")
            L.moe_ep_peer_plan(off_rd, own[rank], W, rank, peer_rows, ROW_BYTES, cap, addr)
            torch.cuda.synchronize()
            got = addr.cpu().numpy().view(np.uint64)
            # the round's pieces at their places; the rest of the rows have no address
            want = np.zeros(rows, np.uint64)
            part = _want_addresses(off_r, off[rank], rank, bases, ROW_BYTES)
            kept_r = off_r[rank, 1:] - off_r[rank, :-1]
            for e in range(N):
                if kept_r[e]:
                    want[off[rank, e]:off[rank, e + 1]] = part[off[rank, e]:off[rank, e + 1]]
            assert np.array_equal(got, want), (r, rank)
            # every address of the round stays inside the receive buffer
            live = got[got != 0]
            dsts = [(a - bases[a // (1 << 36) - 3]) // ROW_BYTES for a in live.astype(object)]
            assert all(0 <= q < cap for q in dsts)
    assert L.moe_device_status() == L.MOE_OK


def test_ep_peer_plan_rows_past_the_buffer_get_no_address():
    W, N = 2, 8
    kept = np.full((W, N), 10)
    off = _offsets(kept)
    off_d = torch.tensor(off, device="cuda")
    peer_rows = torch.tensor([1 << 36, 2 << 36], dtype=torch.int64, device="cuda")
    addr = torch.full((int(off[0, N]),), -1, dtype=torch.int64, device="cuda")
    L.moe_device_status(reset=True)
    L.moe_ep_peer_plan(off_d, off_d[0], W, 0, peer_rows, ROW_BYTES, 50, addr)     # 80 rows go to each rank
    torch.cuda.synchronize()
    got = addr.cpu().numpy().view(np.uint64)
    want = _want_addresses(off, off[0], 0, [1 << 36, 2 << 36], ROW_BYTES)
    inside = [(int(a) - (int(a) >> 36 << 36)) // ROW_BYTES < 50 for a in want]
    assert np.array_equal(got[inside], want[inside])
    assert np.all(got[~np.array(inside)] == 0)
    assert L.moe_device_status(reset=True) == L.MOE_ERR_INVALID_ARG


# ----------------------------------------------------------------------------- kernels, W ranks in one process
@pytest.mark.parametrize("W,d", [(2, 256), (4, 7168)])
def test_ep_peer_dispatch_collect_combine(W, d):
    w = replace(_case(T=257), d=d)
    N, k, T = w.N, w.k, w.T
    El = N // W
    layers, xs = [], []
    shared = make_inputs(w, "cuda", seed=0)
    for r in range(W):
        x = make_inputs(w, "cuda", seed=60 + r, experts=False)["x"]
        lay = MoELayer(w, dict(shared, x=x), "cuda", update_bias=False)
        lay.route(x)
        c = lay.cfg
        L.moe_permute(c, x, lay.topk_idx, lay.counts, lay.offsets, lay.row_of_slot, lay.token_of_row, None,
                      lay.n_dropped, lay.ws)
        layers.append(lay)
        xs.append(x)
    off = torch.stack([lay.offsets for lay in layers])
    off_h = off.cpu().numpy()
    kept = off_h[:, 1:] - off_h[:, :-1]
    cap = int(max(kept[:, dd * El:(dd + 1) * El].sum() for dd in range(W))) + 7
    recv = [torch.full((cap, d), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(W)]
    peer_rows = torch.tensor([b.data_ptr() for b in recv], dtype=torch.int64, device="cuda")
    addrs = []
    for r, lay in enumerate(layers):
        a = torch.zeros(T * k, dtype=torch.int64, device="cuda")
        L.moe_ep_peer_plan(off, lay.offsets, W, r, peer_rows, d * 2, cap, a)
        L.moe_ep_peer_dispatch(lay.cfg, xs[r], lay.row_of_slot, a)
        addrs.append(a)
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    # every receive buffer holds its experts' rows: expert major, then source rank, then row
    tor = [lay.token_of_row.long() for lay in layers]
    for dd in range(W):
        parts = []
        for e in range(dd * El, (dd + 1) * El):
            for s in range(W):
                parts.append(xs[s][tor[s][off_h[s, e]:off_h[s, e + 1]]])
        want = torch.cat(parts)
        n = want.shape[0]
        assert torch.equal(recv[dd][:n], want), dd
        assert torch.isnan(recv[dd][n:].float()).all()           # nothing written past the rows received
    # "results": each destination scales its rows (any per-row function will do here)
    for dd in range(W):
        recv[dd].mul_(2)
    for r, lay in enumerate(layers):
        rows = int(off_h[r, N])
        y_perm = torch.zeros(T * k, d, dtype=torch.bfloat16, device="cuda")
        L.moe_ep_peer_collect(lay.cfg, addrs[r], lay.offsets[N:], y_perm)
        torch.cuda.synchronize()
        assert torch.equal(y_perm[:rows], 2 * xs[r][tor[r][:rows]])
        assert torch.all(y_perm[rows:] == 0)
        # the combine reading the peers' buffers equals moe_combine over the collected rows
        ys = torch.randn(T, d, device="cuda").to(torch.bfloat16)
        y1 = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
        y2 = torch.empty_like(y1)
        L.moe_combine(lay.cfg, y_perm, lay.row_of_slot, lay.topk_w, ys, y1)
        L.moe_combine_peer(lay.cfg, addrs[r], lay.row_of_slot, lay.topk_w, ys, y2)
        torch.cuda.synchronize()
        assert torch.equal(y1, y2), r
    assert L.moe_device_status() == L.MOE_OK


# ----------------------------------------------------------------------------- forward(), W threads
class _Hub:
    def __init__(self, world):
        self.world = world
        self.barrier = threading.Barrier(world, timeout=120)
        self.slot = [None] * world


class _ThreadPeerExchange:
    """The peer-mode exchange interface for W ranks run as threads on one GPU: every
    rank's buffers are plain device buffers of this GPU, and a barrier is an event per
    rank plus a host barrier, each rank's stream then waiting for every rank's event."""

    def __init__(self, hub, rank):
        self.hub, self.rank, self.world = hub, rank, hub.world

    def _post(self, item):
        ev = torch.cuda.Event()
        ev.record()
        self.hub.barrier.wait()
        self.hub.slot[self.rank] = (item, ev)
        self.hub.barrier.wait()
        got = list(self.hub.slot)
        self.hub.barrier.wait()
        for _, e in got:
            torch.cuda.current_stream().wait_event(e)
        return [g[0] for g in got]

    def all_gather(self, t):
        return torch.stack([x.clone() for x in self._post(t)])

    def all_reduce_sum(self, t):
        parts = self._post(t)
        total = torch.stack([p.clone() for p in parts]).sum(0)
        self._post(None)
        t.copy_(total)
        return t

    def barrier(self):
        self._post(None)

    def peer_addresses(self, t):
        return self._post(t.data_ptr())

    def release_peer(self, address):
        pass


@pytest.mark.parametrize("W,recv_factor,device_plan", [(2, 4.0, False), (4, 1.0, False), (2, 0.4, False),
                                                        (2, 1.0, True), (4, 1.0, True)])
def test_ep_peer_forward_threads_matches_single_rank(W, recv_factor, device_plan):
    w = _case()
    shared = make_inputs(w, "cuda", seed=0)
    xs = [make_inputs(w, "cuda", seed=80 + r, experts=False)["x"] for r in range(W)]
    bias0 = shared["bias"].clone()
    hub = _Hub(W)
    weights = [dict(shared, bias=bias0.clone()) for _ in range(W)]
    layers = [EPMoELayer(w, weights[r], r, W, "cuda", exchange=_ThreadPeerExchange(hub, r), update_bias=True,
                         recv_factor=recv_factor, peer=True, device_plan=device_plan) for r in range(W)]
    ys, errs = [None] * W, []

    def run(r):
        try:
            with torch.cuda.stream(torch.cuda.Stream()):
                for _ in range(2):                              # the second forward reuses the mapped buffers
                    weights[r]["bias"].copy_(bias0)
                    ys[r] = layers[r].forward(xs[r]).clone()
                torch.cuda.current_stream().synchronize()
        except Exception as e:          # reported below
            errs.append(e)
            hub.barrier.abort()

    th = [threading.Thread(target=run, args=(r,)) for r in range(W)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errs, errs
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    R = 1 if device_plan else len(layers[0].plans)
    if device_plan:
        assert layers[0].recv_cap == W * w.T * min(w.k, w.N // W) and not layers[0].plans
    if recv_factor >= 4.0:
        assert R == 1                                   # the combine reads the peers' buffers
    if recv_factor < 1.0 and not device_plan:
        assert R > 1                                    # every round's results are collected
    assert layers[0].fuse_shared
    counts = torch.zeros(w.N, dtype=torch.int64, device="cuda")
    for r in range(W):
        single = MoELayer(w, dict(shared, x=xs[r], bias=bias0.clone()), "cuda", update_bias=False)
        y_ref = single.forward(xs[r])
        torch.cuda.synchronize()
        assert torch.equal(ys[r][:w.T], y_ref[:w.T]), r
        counts += single.counts.long()
    ref_bias = O.bias_update(bias0.double().cpu().numpy(), counts.cpu().numpy(), rate=w.bias_rate)
    for r in range(W):
        assert np.max(np.abs(weights[r]["bias"].double().cpu().numpy() - ref_bias)) < 1e-7
    # rank 0's output against the oracle's layer forward on its tokens (dropless: tokens are
    # independent), within the bf16 bar on the tokens whose expert choice is clear
    out = O.layer_forward(f64(xs[0]), f64(shared["w_gate"]), oracle_cfg(w), expert_weights_fn(shared),
                          shared_weights(shared), bias=f64(bias0))
    clear = out["routing"]["margin"] >= NEAR_TIE
    assert clear.mean() > 0.95
    assert np.array_equal(i64(layers[0].base.topk_idx)[clear], out["routing"]["idx"][clear])
    assert rel_err(f64(ys[0][:w.T])[clear], out["y"][clear]) < TOL_BF16


@pytest.mark.parametrize("device_plan", [False, True])
def test_ep_peer_forward_one_rank_receives_nothing(device_plan):
    """A selection bias that sends every token to rank 0's experts: rank 1's experts get no
    rows (an empty grouped FFN), rank 1's combine reads every result from rank 0's buffer,
    and both ranks still equal the single-rank layer."""
    import threading
    W = 2
    w = _case()
    shared = make_inputs(w, "cuda", seed=0)
    El = w.N // W
    bias = torch.zeros_like(shared["bias"])
    bias[:El] = 10.0                                   # experts of rank 0 win every selection
    xs = [make_inputs(w, "cuda", seed=120 + r, experts=False)["x"] for r in range(W)]
    hub = _Hub(W)
    weights = [dict(shared, bias=bias.clone()) for _ in range(W)]
    layers = [EPMoELayer(w, weights[r], r, W, "cuda", exchange=_ThreadPeerExchange(hub, r), update_bias=False,
                         peer=True, device_plan=device_plan) for r in range(W)]
    ys, errs = [None] * W, []

    def run(r):
        try:
            with torch.cuda.stream(torch.cuda.Stream()):
                ys[r] = layers[r].forward(xs[r]).clone()
                torch.cuda.current_stream().synchronize()
        except Exception as e:          # reported below
            errs.append(e)
            hub.barrier.abort()

    th = [threading.Thread(target=run, args=(r,)) for r in range(W)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errs, errs
    torch.cuda.synchronize()
    assert L.moe_device_status() == L.MOE_OK
    assert int(layers[1].local_offsets[0][El].item()) == 0      # rank 1 computed nothing
    assert torch.all(layers[0].base.topk_idx < El) and torch.all(layers[1].base.topk_idx < El)
    for r in range(W):
        single = MoELayer(w, dict(shared, x=xs[r], bias=bias.clone()), "cuda", update_bias=False)
        y_ref = single.forward(xs[r])
        torch.cuda.synchronize()
        assert torch.equal(ys[r][:w.T], y_ref[:w.T]), r


# ----------------------------------------------------------------------------- two processes, CUDA IPC
def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _GlooHostExchange:
    """The peer-mode exchange for processes sharing one GPU: collectives on the host
    (gloo), each preceded by a device synchronisation, so a barrier orders every
    process's device work without any kernel waiting for another process."""

    def __init__(self):
        import torch.distributed as dist
        self.dist = dist
        self.rank, self.world = dist.get_rank(), dist.get_world_size()

    def _sync(self):
        torch.cuda.synchronize()
        self.dist.barrier()

    def all_gather(self, t):
        self._sync()
        c = t.cpu().contiguous()
        out = [torch.empty_like(c) for _ in range(self.world)]
        self.dist.all_gather(out, c)
        return torch.stack(out).to(t.device)

    def all_reduce_sum(self, t):
        self._sync()
        c = t.cpu().contiguous()
        self.dist.all_reduce(c)
        t.copy_(c)
        return t

    def barrier(self):
        self._sync()

    def peer_addresses(self, t):
        self._sync()
        hs = [None] * self.world
        self.dist.all_gather_object(hs, L.moe_peer_export(t))
        return [t.data_ptr() if r == self.rank else L.moe_peer_import(hs[r]) for r in range(self.world)]

    def release_peer(self, address):
        L.moe_peer_close(address)


def _ipc_worker(rank, port, out_dir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=2)
    try:
        torch.cuda.set_device(0)
        ex = _GlooHostExchange()
        # the mapping alone: read the other process's buffer through its imported address
        mine = torch.full((64, 256), float(rank + 1), dtype=torch.bfloat16, device="cuda")
        mine_off = torch.empty(300, 256, dtype=torch.bfloat16, device="cuda")[100:164]   # inside an allocation
        mine_off.fill_(float(10 + rank))
        a_full = ex.peer_addresses(mine)
        a_off = ex.peer_addresses(mine_off)
        other = 1 - rank
        cfg_w = replace(_case(T=8), d=256)
        lay0 = MoELayer(cfg_w, make_inputs(cfg_w, "cuda", seed=0), "cuda", update_bias=False)
        got = torch.zeros(2, 256, dtype=torch.bfloat16, device="cuda")
        addr = torch.tensor([a_full[other], a_off[other]], dtype=torch.int64, device="cuda")
        n = torch.tensor([2], dtype=torch.int32, device="cuda")
        L.moe_ep_peer_collect(lay0.cfg, addr, n, got)
        torch.cuda.synchronize()
        ok_map = bool(torch.all(got[0] == other + 1)) and bool(torch.all(got[1] == 10 + other))
        ex.barrier()
        for a in (a_full[other], a_off[other]):
            L.moe_peer_close(a)
        # the peer forward, twice
        w = _case()
        shared = make_inputs(w, "cuda", seed=0)
        x = make_inputs(w, "cuda", seed=90 + rank, experts=False)["x"]
        single = MoELayer(w, dict(shared, x=x), "cuda", update_bias=False)
        y_ref = single.forward(x).clone()
        torch.cuda.synchronize()
        ok_fwd = True
        for device_plan in (False, True):
            lay = EPMoELayer(w, shared, rank, 2, "cuda", exchange=ex, update_bias=False, recv_factor=1.0, peer=True,
                             device_plan=device_plan)
            for _ in range(2):
                y = lay.forward(x).clone()
            torch.cuda.synchronize()
            ok_fwd = ok_fwd and bool(torch.equal(y[:w.T], y_ref[:w.T]))
            ex.barrier()
            lay.close()
            ex.barrier()
        status = L.moe_device_status()
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), ok_map=ok_map, ok_fwd=ok_fwd, status=status)
    finally:
        dist.destroy_process_group()


def test_ep_peer_two_processes_ipc(tmp_path):
    import torch.multiprocessing as mp
    mp.start_processes(_ipc_worker, args=(_free_port(), str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    for r in range(2):
        z = np.load(tmp_path / f"r{r}.npz")
        assert bool(z["ok_map"]), r
        assert bool(z["ok_fwd"]), r
        assert int(z["status"]) == L.MOE_OK
