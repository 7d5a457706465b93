"""The allocation-free permutation entry point against the regular one.

moe_permute_noalloc serves callers that cannot allocate device memory (a
plugin inside an application whose memory pool owns the device, or a static
memory plan): it keeps its scratch in a fixed array inside the library.  Its
outputs must equal moe_permute's exactly (they are integer maps and a byte
copy), on two calls in a row, since every call reuses the same array.  This file
is collected last so that a failure here cannot hide the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_21_b200 import _lib as L
from sparse_mixture_experts_21_b200.layer import make_config
from sparse_mixture_experts_21_b200.synth import WORKLOADS, random_routing
from tests.parity_util import oracle_cfg

pytestmark = pytest.mark.gpu


def _buffers(w):
    T, k, N = w.T, w.k, w.N
    dev = "cuda"
    i32 = lambda *s: torch.full(s, -5, dtype=torch.int32, device=dev)  # noqa: E731
    return {"counts": i32(N), "offsets": i32(N + 1), "ros": i32(T, k), "tor": i32(T * k),
            "nd": i32(2), "xp": torch.zeros(T * k, w.d, dtype=torch.bfloat16, device=dev)}


@pytest.mark.parametrize("name,T,seed", [("deepseek_v3", 16384, 11), ("switch_skewed", 20000, 12)])
def test_noalloc_matches_permute_twice(name, T, seed):
    from dataclasses import replace
    w = replace(WORKLOADS[name], T=T, d=256)
    c = make_config(w)
    g = torch.Generator(device="cuda").manual_seed(seed)
    ws = torch.empty(max(L.workspace_size(c), 16), dtype=torch.uint8, device="cuda")
    for call in range(2):      # the second call reuses the array the first one left behind
        x = torch.randn(T, w.d, generator=g, device="cuda").to(torch.bfloat16)
        idx = random_routing(T, w.N, w.k, "cuda", seed=seed + call, hot=3 if call else None)
        ref, got = _buffers(w), _buffers(w)
        L.moe_permute(c, x, idx, ref["counts"], ref["offsets"], ref["ros"], ref["tor"], ref["xp"],
                      ref["nd"], ws)
        L.moe_permute_noalloc(c, x, idx, got["counts"], got["offsets"], got["ros"], got["tor"],
                              got["xp"], got["nd"])
        torch.cuda.synchronize()
        for key in ref:
            assert torch.equal(ref[key], got[key]), f"call {call}: {key} differs"
        # and against the oracle's permutation of the same routing
        p = O.permutation(idx.cpu().numpy().astype(np.int64), w.N, O.capacity(oracle_cfg(w), T))
        assert np.array_equal(got["counts"].cpu().numpy(), p["counts"])
        assert np.array_equal(got["offsets"].cpu().numpy(), p["offsets"])
        assert np.array_equal(got["ros"].cpu().numpy(), p["row_of_slot"])
        assert np.array_equal(got["tor"].cpu().numpy()[:p["R"]], p["token_of_row"])
        assert got["nd"].cpu().tolist() == [p["dropped_slots"], p["dropped_tokens"]]


def test_noalloc_without_gather():
    """x_perm = NULL skips the row gather, as in moe_permute (x may then be NULL)."""
    from dataclasses import replace
    w = replace(WORKLOADS["deepseek_v3"], T=3000, d=256)
    c = make_config(w)
    idx = random_routing(w.T, w.N, w.k, "cuda", seed=13)
    ws = torch.empty(max(L.workspace_size(c), 16), dtype=torch.uint8, device="cuda")
    ref, got = _buffers(w), _buffers(w)
    L.moe_permute(c, None, idx, ref["counts"], ref["offsets"], ref["ros"], ref["tor"], None, ref["nd"], ws)
    L.moe_permute_noalloc(c, None, idx, got["counts"], got["offsets"], got["ros"], got["tor"], None, got["nd"])
    torch.cuda.synchronize()
    for key in ("counts", "offsets", "ros", "tor", "nd"):
        assert torch.equal(ref[key], got[key]), key
    assert torch.all(got["xp"] == 0)


def test_noalloc_rejects_sizes_beyond_its_array():
    w = WORKLOADS["deepseek_v3"]
    c = make_config(w, T=300000)          # ceil(300000 / 256) * 256 > 262144 entries
    st = L.load().moe_permute_noalloc(ctypes.byref(c), 0x1000000, 0x1000000, 0x1000000, 0x1000000,
                                      0x1000000, 0x1000000, 0x1000000, 0x1000000, None)
    assert st == L.MOE_ERR_WORKSPACE_TOO_SMALL
