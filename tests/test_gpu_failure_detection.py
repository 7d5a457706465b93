"""Device-side failure detection without a GPU fault: a bounded wait that can never
complete gives up, records MOE_ERR_DEVICE_TIMEOUT in the device status word, and
leaves the context usable (the next layer forward still runs and is correct)."""
import time

import pytest
import torch

from sparse_mixture_experts_21_b200 import _lib as L
from sparse_mixture_experts_21_b200.layer import MoELayer
from sparse_mixture_experts_21_b200.synth import WORKLOADS, make_inputs
from dataclasses import replace

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    w = replace(WORKLOADS["deepseek_v3"], T=256, d=512, N=64, f=256, f_shared=256)
    inp = make_inputs(w, "cuda")
    lay = MoELayer(w, inp, "cuda", update_bias=False)
    before = lay.forward(inp["x"]).clone()
    assert L.moe_device_status(reset=True) == L.MOE_OK
    flag = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    t0 = time.time()
    L.moe_selftest_wait_timeout(200_000_000, flag)          # ~0.1 s at the B200 clock
    torch.cuda.synchronize()
    assert time.time() - t0 < 30
    assert int(flag.item()) == 0                             # the wait gave up ...
    assert L.moe_device_status(reset=True) == L.MOE_ERR_DEVICE_TIMEOUT   # ... and said so
    assert L.moe_device_status(reset=False) == L.MOE_OK      # cleared by the reset
    after = lay.forward(inp["x"])                            # the context is still usable
    torch.cuda.synchronize()
    assert torch.equal(before, after)
    assert L.moe_device_status() == L.MOE_OK


def test_selftest_rejects_bad_limits():
    lib = L.load()
    assert lib.moe_selftest_wait_timeout(0, None, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_selftest_wait_timeout(10 ** 12, None, None) == L.MOE_ERR_INVALID_ARG
