"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
symbol the header declares, answers sizing queries, and rejects bad arguments
before enqueueing anything."""
import ctypes
import os
import re

import pytest

from sparse_mixture_experts_21_b200 import _lib as L
from sparse_mixture_experts_21_b200 import layer, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    inc = os.path.join(ROOT, "include")
    for fn in os.listdir(inc):
        if fn.endswith(".h"):
            text = open(os.path.join(inc, fn)).read()
            names.update(re.findall(r"^\s*(?:int|const char\*)\s+(moe_\w+)\s*\(", text, re.M))
    return names


def test_library_exports_every_declared_symbol(lib):
    declared = _declared_symbols()
    assert declared >= set(L.EXPORTED)
    for name in declared:
        assert getattr(lib, name) is not None


def test_header_is_plain_c(tmp_path):
    """include/moe_b200.h compiles as strict C99 and as C++ (plain pointers and sizes, no
    torch or CUDA types in the signatures)."""
    import shutil
    import subprocess
    src = tmp_path / "use_header.c"
    src.write_text('#include "moe_b200.h"\nint main(void) { return 0; }\n')
    inc = os.path.join(ROOT, "include")
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only", "-I", inc,
                    str(src)], check=True)
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Werror", "-fsyntax-only", "-I", inc, "-x", "c++", str(src)],
                   check=True)


def test_config_struct_layout():
    assert ctypes.sizeof(L.MoeConfig) == 64
    assert L.MoeConfig.capacity_factor.offset == 56
    assert ctypes.sizeof(L.MoeStats) == 64
    assert L.MoeStats.near_ties.offset == 44 and L.MoeStats.T.offset == 48


@pytest.mark.parametrize("T,N,k,cf", [(8192, 64, 6, 1.0), (1000, 7, 3, 1.25), (5, 64, 6, 1.0), (300, 4, 4, 2.0),
                                      (4097, 96, 2, 0.8)])
def test_expert_choice_capacity_matches_oracle(lib, T, N, k, cf):
    """The library's expert-choice capacity (host only) against the oracle's reading,
    C = min(T, ceil(cf k T / N))."""
    from oracle import moe_oracle as O
    w = synth.WORKLOADS["ec_deepseekmoe_16b"]
    c = layer.make_config(w, T=T)
    c.n_experts, c.top_k, c.capacity_factor = N, k, cf
    assert L.expert_choice_capacity(c) == O.expert_choice_capacity(N, k, T, cf)
    c.capacity_factor = 0.0
    out = ctypes.c_int32()
    assert lib.moe_expert_choice_capacity(ctypes.byref(c), ctypes.byref(out)) == L.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_sizing_queries(lib, name):
    w = synth.WORKLOADS[name]
    c = layer.make_config(w)
    if w.dtype == "bf16" and w.N <= 256:          # tensor-core router: 128 tokens per block
        tm = 128
        np_ = max(16, 1 << (w.N - 1).bit_length())
        route_ws = np_ * 3 * (-(-w.d // 64) * 64) * 2
    else:
        tm = 32 if w.N <= 32 or w.N > 256 else 64
        route_ws = 0
    assert L.route_partials(c) == (w.T + tm - 1) // tm
    assert L.workspace_size(c) == max(((w.T + 255) // 256) * w.N * 4, route_ws)
    cap = L.capacity(c)
    if w.capacity == "dropless":
        assert cap == 2 ** 63 - 1
    else:
        assert cap == -(-int(w.cf * w.T) // w.N)


def test_capacity_variants(lib):
    c = layer.make_config(synth.WORKLOADS["tiny_top2_fp32"])
    assert L.capacity(c) == 40                        # ceil(1.25 * 256 / 8)
    c.capacity_mode = L.CAP_CF_K_T_OVER_N_FLOOR
    assert L.capacity(c) == 80                        # max(int(2 * 256 / 8 * 1.25), 2)
    c.T, c.capacity_factor = 10, 0.01
    assert L.capacity(c) == 2                         # never below k


def _status(fn, *args):
    return fn(*args)


@pytest.mark.parametrize("field,value", [
    ("top_k", 0), ("top_k", 9), ("n_experts", 0), ("n_experts", 513), ("d_model", 12),
    ("score_fn", 7), ("x_dtype", 5), ("capacity_mode", 9), ("n_groups", 3),
])
def test_invalid_config_rejected(lib, field, value):
    c = layer.make_config(synth.WORKLOADS["tiny_top2_fp32"])
    setattr(c, field, value)
    out = ctypes.c_int64()
    assert lib.moe_capacity(ctypes.byref(c), ctypes.byref(out)) == L.MOE_ERR_INVALID_ARG


def test_group_limit_validation(lib):
    c = layer.make_config(synth.WORKLOADS["deepseek_v3"])
    out = ctypes.c_int64()
    assert lib.moe_capacity(ctypes.byref(c), ctypes.byref(out)) == L.MOE_OK
    c.topk_groups = 0
    assert lib.moe_capacity(ctypes.byref(c), ctypes.byref(out)) == L.MOE_ERR_INVALID_ARG
    c.topk_groups, c.group_score_topn = 4, 33              # more than a group holds
    assert lib.moe_capacity(ctypes.byref(c), ctypes.byref(out)) == L.MOE_ERR_INVALID_ARG
    c.group_score_topn, c.n_groups, c.topk_groups = 2, 32, 1   # 1 group of 8 < k = 8? equal: ok
    assert lib.moe_capacity(ctypes.byref(c), ctypes.byref(out)) == L.MOE_OK
    c.top_k = 9
    assert lib.moe_capacity(ctypes.byref(c), ctypes.byref(out)) == L.MOE_ERR_INVALID_ARG


def test_null_and_misaligned_pointers_rejected(lib):
    c = layer.make_config(synth.WORKLOADS["tiny_top2_fp32"])
    cp = ctypes.byref(c)
    # null required pointers: rejected on the host, nothing launched
    assert lib.moe_route(cp, None, None, None, None, None, None, None, None, None, None, None, 0, None) == \
        L.MOE_ERR_INVALID_ARG
    bad = 0x1000008  # not 16-byte aligned
    ok = 0x1000000
    assert lib.moe_route(cp, bad, ok, None, None, ok, ok, ok, ok, None, None, None, 0, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(cp, ok, ok, ok, None, None, bad, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_grouped_ffn(cp, ok, 10, ok, 0, ok, ok, ok, 256, ok, ok, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_grouped_ffn(cp, ok, 10, ok, 1, ok, ok, ok, 12, ok, ok, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_bias_update(cp, None, ok, 1e-3, 0.0, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_router_stats(cp, ok, ok, ok, ok, ok, None, 1e-4, None, 0.0, 0.0, None, None, None, None) == \
        L.MOE_ERR_INVALID_ARG
    assert lib.moe_router_stats_partial(cp, ok, ok, ok, ok, ok, None, 1e-4, None, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_router_stats_partial(cp, ok, ok, ok, ok, ok, None, 1e-4, ok + 4, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_router_stats_finalize(cp, None, None, 0.0, 0.0, ok, None, None, None, None) == \
        L.MOE_ERR_INVALID_ARG


def test_gathering_ffn_checks(lib):
    """moe_grouped_ffn_gather: bf16 with d % 64 == 0 only; its row map is required; the
    shared weights come all three or not at all; no rows or no tokens is a no-op.
    Nothing here reaches the GPU."""
    ok, UN, IA = 0x1000000, L.MOE_ERR_UNSUPPORTED, L.MOE_ERR_INVALID_ARG
    c = layer.make_config(synth.WORKLOADS["deepseek_v3"])
    cp = ctypes.byref(c)
    no = (None, None, None)

    def f(*a, shared=no):
        return lib.moe_grouped_ffn_gather(*a, *shared, None)
    assert f(cp, ok, 100, None, 800, ok, 256, ok, ok, ok, 2048, ok, ok) == IA      # token_of_row
    assert f(cp, ok, 100, ok + 2, 800, ok, 256, ok, ok, ok, 2048, ok, ok) == IA    # misaligned map
    assert f(cp, ok + 8, 100, ok, 800, ok, 256, ok, ok, ok, 2048, ok, ok) == IA    # misaligned x
    assert f(cp, ok, -1, ok, 800, ok, 256, ok, ok, ok, 2048, ok, ok) == IA
    assert f(cp, ok, 100, ok, 800, ok, 0, ok, ok, ok, 2048, ok, ok) == IA          # G
    assert f(cp, ok, 100, ok, 800, ok, 512, ok, ok, ok, 2048, ok, ok) == IA        # G: one slot for the shared
    assert f(cp, ok, 100, ok, 800, ok, 256, ok, ok, ok, 2047, ok, ok) == IA        # f % 8
    assert f(cp, ok, 100, ok, 800, ok, 256, ok, ok, ok, 2048, ok, ok, shared=(ok, None, ok)) == IA
    assert f(cp, ok, 100, ok, 800, ok, 256, ok, ok, ok, 2048, ok, ok, shared=(ok, ok, ok + 8)) == IA
    assert f(cp, None, 0, ok, 800, ok, 256, None, None, None, 2048, None, None) == L.MOE_OK
    assert f(cp, None, 100, ok, 0, ok, 256, None, None, None, 2048, None, None) == L.MOE_OK
    c32 = layer.make_config(synth.WORKLOADS["tiny_top2_fp32"])
    assert f(ctypes.byref(c32), ok, 10, ok, 20, ok, 8, ok, ok, ok, 256, ok, ok) == UN
    c.d_model = 7168 + 8                                                                    # d % 64 != 0
    assert f(cp, ok, 100, ok, 800, ok, 256, ok, ok, ok, 2048, ok, ok) == UN


def test_ffn_pass_entry_checks(lib):
    """moe_grouped_ffn_gate_up / moe_grouped_ffn_down: bf16 only, G and f in range, the
    shared rows only with their weights; no rows is a no-op.  Nothing here reaches the GPU."""
    ok, UN, IA = 0x1000000, L.MOE_ERR_UNSUPPORTED, L.MOE_ERR_INVALID_ARG
    c = layer.make_config(synth.WORKLOADS["deepseek_v3"])
    cp = ctypes.byref(c)
    gu, dn = lib.moe_grouped_ffn_gate_up, lib.moe_grouped_ffn_down
    assert gu(cp, ok, 100, ok, 0, ok, ok, 2048, ok, None) == IA             # G
    assert gu(cp, ok, 100, ok, 513, ok, ok, 2048, ok, None) == IA
    assert gu(cp, ok, 100, ok, 4, ok, ok, 2047, ok, None) == IA             # f % 8
    assert gu(cp, ok + 8, 100, ok, 4, ok, ok, 2048, ok, None) == IA         # misaligned rows
    assert gu(cp, None, 0, ok, 4, None, None, 2048, None, None) == L.MOE_OK
    assert dn(cp, ok, 100, ok, 512, ok, 2048, ok, 0, None, None) == IA      # G: one slot for the shared
    assert dn(cp, ok, 100, ok, 4, ok, 2048, ok, 10, None, None) == IA       # shared rows without ws2
    assert dn(cp, ok, 100, ok, 4, ok, 2048, ok, 0, ok, None) == IA          # ws2 without shared rows
    assert dn(cp, ok, 100, ok, 4, ok, 2048, ok, -1, None, None) == IA
    assert dn(cp, ok, 100, ok, 4, ok, 2048, ok + 4, 0, None, None) == IA    # misaligned y
    assert dn(cp, None, 0, ok, 4, None, 2048, None, 0, None, None) == L.MOE_OK
    c32 = layer.make_config(synth.WORKLOADS["tiny_top2_fp32"])
    assert gu(ctypes.byref(c32), ok, 10, ok, 8, ok, ok, 256, ok, None) == UN
    assert dn(ctypes.byref(c32), ok, 10, ok, 8, ok, 256, ok, 0, None, None) == UN


def test_fused_shared_ffn_checks(lib):
    """moe_grouped_ffn_shared: bf16 only, G <= 511, every buffer present and aligned;
    no shared rows is moe_grouped_ffn.  Nothing here reaches the GPU."""
    ok, UN, IA = 0x1000000, L.MOE_ERR_UNSUPPORTED, L.MOE_ERR_INVALID_ARG
    c = layer.make_config(synth.WORKLOADS["deepseek_v3"])
    cp = ctypes.byref(c)
    f = lib.moe_grouped_ffn_shared
    good = [ok, 800, ok, 256, ok, ok, ok, 2048, ok, ok, ok, 100, ok, ok, ok, None]
    def call(**kw):
        a = list(good)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return f(cp, *a)
    assert call(a3=512) == IA                       # G: one slot is the shared group
    assert call(a3=0) == IA
    assert call(a11=-1) == IA                       # T
    assert call(a12=None) == IA                     # ws1
    assert call(a10=ok + 4) == IA                   # x misaligned
    assert call(a8=None) == IA                      # h_scratch
    assert call(a1=(1 << 31) - 50) == UN            # rows_cap + T past INT32_MAX
    assert call(a7=2047) == IA                      # f % 8
    c32 = layer.make_config(synth.WORKLOADS["tiny_top2_fp32"])
    assert f(ctypes.byref(c32), *good) == UN
    # T = 0 with nothing to do: the plain grouped FFN's no-op
    assert f(cp, None, 0, ok, 1, None, None, None, 256, None, None, None, 0, None, None, None, None) == L.MOE_OK


def test_nvfp4_argument_checks(lib):
    """NVFP4 entry points reject bad shapes, missing tensor scales and unsupported
    configurations before anything reaches the GPU."""
    ok, UN, IA = 0x1000000, L.MOE_ERR_UNSUPPORTED, L.MOE_ERR_INVALID_ARG
    q = lib.moe_quantize_nvfp4
    assert q(ok, 128, 96, 0, ok, ok, None, None) == IA           # cols % 64
    assert q(ok, 130, 128, 64, ok, ok, ok, None) == IA           # rows % tensor_rows
    assert q(ok, 128, 128, 64, ok, ok, None, None) == IA         # tensor scales need g
    assert q(ok, 128, 128, 0, ok + 2, ok, None, None) == IA      # codes 4-byte aligned
    assert q(ok, 0, 128, 0, None, None, None, None) == L.MOE_OK  # nothing to do
    c = layer.make_config(synth.WORKLOADS["deepseek_v3"])
    cp = ctypes.byref(c)
    ffn = lib.moe_grouped_ffn_nvfp4
    args = [ok, ok, 1024, ok, 4, ok, ok, ok, ok, ok, ok, ok, ok, ok, 2048, ok, ok, ok, None]
    assert ffn(cp, *args[:14], 2176, *args[15:]) == UN             # f % 256
    assert ffn(cp, *args[:4], 0, *args[5:]) == IA                  # G
    assert ffn(cp, *args[:7], None, *args[8:]) == IA               # g1
    c32 = layer.make_config(synth.WORKLOADS["tiny_top2_fp32"])
    assert ffn(ctypes.byref(c32), *args) == UN
    assert lib.moe_permute_nvfp4(ctypes.byref(c32), ok, ok, ok, ok, ok, ok, None, None, None) == UN
    assert lib.moe_permute_nvfp4(cp, ok, ok, None, ok, ok, ok, None, None, None) == IA   # no row maps, no q


def test_route_prepare_checks(lib):
    ok = 0x1000000
    c = layer.make_config(synth.WORKLOADS["deepseek_v3"])
    assert L.route_prepare_size(c) == L.workspace_size(c) or L.route_prepare_size(c) <= L.workspace_size(c)
    assert lib.moe_route_prepare(ctypes.byref(c), ok, ok, 16, None) == L.MOE_ERR_WORKSPACE_TOO_SMALL
    assert lib.moe_route_prepare(ctypes.byref(c), None, ok, 1 << 30, None) == L.MOE_ERR_INVALID_ARG
    cf = layer.make_config(synth.WORKLOADS["tiny_top2_fp32"])          # fp32 router: no split
    assert L.route_prepare_size(cf) == 0
    assert lib.moe_route_prepare(ctypes.byref(cf), ok, ok, 1 << 30, None) == L.MOE_ERR_UNSUPPORTED
    # a NULL router weight is only accepted where a prepared split exists
    assert lib.moe_route(ctypes.byref(cf), ok, None, None, None, ok, ok, ok, ok, None, None, None, 0, None) == \
        L.MOE_ERR_INVALID_ARG


def test_workspace_too_small_rejected(lib):
    c = layer.make_config(synth.WORKLOADS["tiny_top2_fp32"])
    ok = 0x1000000
    st = lib.moe_permute(ctypes.byref(c), ok, ok, ok, ok, ok, ok, ok, ok, ok, 4, None)
    assert st == L.MOE_ERR_WORKSPACE_TOO_SMALL
    c3 = layer.make_config(synth.WORKLOADS["deepseek_v3"])
    st = lib.moe_route(ctypes.byref(c3), ok, ok, None, None, ok, ok, ok, ok, None, None, ok, 1024, None)
    assert st == L.MOE_ERR_WORKSPACE_TOO_SMALL


def test_empty_batch_is_a_no_op(lib):
    c = layer.make_config(synth.WORKLOADS["tiny_top2_fp32"], T=0)
    assert lib.moe_route(ctypes.byref(c), None, None, None, None, None, None, None, None, None, None, None, 0,
                         None) == L.MOE_OK
    assert lib.moe_combine(ctypes.byref(c), None, None, None, None, None, None, None) == L.MOE_OK
    assert lib.moe_grouped_ffn(ctypes.byref(c), None, 0, 0x1000000, 1, None, None, None, 256, None, None,
                               None) == L.MOE_OK


def test_variant_argument_checks(lib):
    c = layer.make_config(synth.WORKLOADS["deepseekmoe_16b"])
    ok = 0x1000000
    c.shared_sink = 1          # the sink needs its shared-weight output
    assert lib.moe_route(ctypes.byref(c), ok, ok, None, None, ok, ok, ok, ok, None, None, ok, 1 << 30,
                         None) == L.MOE_ERR_INVALID_ARG
    c.shared_sink = 2
    assert lib.moe_capacity(ctypes.byref(c), ctypes.byref(ctypes.c_int64())) == L.MOE_ERR_INVALID_ARG
    c.shared_sink = 0
    assert lib.moe_bias_update_ema(ctypes.byref(c), ok, ok, 1.0, ok, 1e-3, 0.0, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_bias_update_seq(ctypes.byref(c), ok, ok, 4, ok, 1e-3, 0.0, ok, 8, None) == \
        L.MOE_ERR_WORKSPACE_TOO_SMALL


def test_status_strings(lib):
    for s in range(6):
        assert lib.moe_status_string(s)
    assert b"timed out" in lib.moe_status_string(L.MOE_ERR_DEVICE_TIMEOUT)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(FileNotFoundError):
        L.load(str(tmp_path / "nope.so"))


def test_low_precision_argument_checks(lib):
    """FP8 / MXFP8 entry points reject bad shapes and pointers before touching the GPU."""
    ok = 0x1000000
    IA, UN = L.MOE_ERR_INVALID_ARG, L.MOE_ERR_UNSUPPORTED
    # block quantisation: cols must be a multiple of 128, block rows 1 or 128
    assert lib.moe_quantize_fp8(ok, 10, 100, 1, ok, ok, None) == IA
    assert lib.moe_quantize_fp8(ok, 10, 128, 64, ok, ok, None) == IA
    assert lib.moe_quantize_fp8(ok + 8, 10, 128, 1, ok, ok, None) == IA       # misaligned x
    assert lib.moe_quantize_fp8(ok, 0, 128, 1, None, None, None) == L.MOE_OK  # nothing to do
    assert lib.moe_quantize_mxfp8(ok, 10, 96, ok, ok, None) == IA             # MXFP8 wants cols % 128
    assert lib.moe_quantize_mxfp8(ok, 10, 128, ok + 4, ok, None) == IA        # codes not 8-byte aligned
    c = layer.make_config(synth.WORKLOADS["deepseek_v3"])
    # grouped FFNs: f % 128, G range, fp32 configs unsupported
    args = (ok, ok, 1024, ok, 4, ok, ok, ok, ok, ok, ok)
    assert lib.moe_grouped_ffn_fp8(ctypes.byref(c), *args, 2000, ok, ok, ok, None) == UN
    assert lib.moe_grouped_ffn_mxfp8(ctypes.byref(c), *args, 2000, ok, ok, ok, None) == UN
    assert lib.moe_grouped_ffn_mxfp8(ctypes.byref(c), ok, ok, 1024, ok, 0, ok, ok, ok, ok, ok, ok, 2048, ok, ok,
                                     ok, None) == IA
    assert lib.moe_grouped_ffn_mxfp8(ctypes.byref(c), ok, ok + 4, 1024, ok, 4, ok, ok, ok, ok, ok, ok, 2048, ok,
                                     ok, ok, None) == IA                      # scale atoms 16-byte aligned
    c32 = layer.make_config(synth.WORKLOADS["tiny_top2_fp32"])
    assert lib.moe_grouped_ffn_fp8(ctypes.byref(c32), ok, ok, 64, ok, 1, ok, ok, ok, ok, ok, ok, 256, ok, ok, ok,
                                   None) == UN
    # the quantising permutations need their row maps
    assert lib.moe_permute_mxfp8(ctypes.byref(c), ok, None, ok, ok, ok, ok, None, None, None) == IA
    assert lib.moe_permute_fp8(ctypes.byref(c), ok, ok, None, ok, None, None, None) == IA


def test_expert_parallel_argument_checks(lib):
    ok = 0x1000000
    IA = L.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_plan(ok, 3, 0, 256, ok, ok, ok, ok, 10, None) == IA    # 256 experts over 3 ranks
    assert lib.moe_ep_plan(ok, 4, 4, 256, ok, ok, ok, ok, 10, None) == IA    # rank out of range
    assert lib.moe_ep_plan(None, 4, 0, 256, ok, ok, ok, ok, 10, None) == IA
    assert lib.moe_rows_move(ok, 24, ok, None, 10, 0, ok, None) == IA        # rows of 24 bytes
    assert lib.moe_rows_move(ok, 32, ok, None, 10, 2, ok, None) == IA        # bad direction flag
    assert lib.moe_rows_move(ok, 32, ok, None, 0, 0, ok, None) == L.MOE_OK   # no rows


def test_peer_exchange_argument_checks(lib):
    """The peer-memory exchange entry points reject bad arguments before any CUDA call."""
    ok = 0x1000000
    IA = L.MOE_ERR_INVALID_ARG
    c = layer.make_config(synth.WORKLOADS["deepseek_v3"])
    handle = ctypes.create_string_buffer(L.PEER_HANDLE_BYTES)
    out = ctypes.c_void_p()
    assert lib.moe_peer_export(None, handle) == IA
    assert lib.moe_peer_export(ok, None) == IA
    assert lib.moe_peer_import(None, ctypes.byref(out)) == IA
    assert lib.moe_peer_import(handle, None) == IA
    neg = ctypes.create_string_buffer(b"\0" * 64 + (-16).to_bytes(8, "little", signed=True), L.PEER_HANDLE_BYTES)
    assert lib.moe_peer_import(neg, ctypes.byref(out)) == IA                  # negative offset
    assert lib.moe_peer_close(None) == IA
    assert lib.moe_peer_close(ok) == IA                                       # never imported
    # plan: W must divide N, rank in range, rows a multiple of 16 bytes, every pointer given
    assert lib.moe_ep_peer_plan(ok, ok, 3, 0, 256, ok, 14336, 100, ok, None) == IA
    assert lib.moe_ep_peer_plan(ok, ok, 4, -1, 256, ok, 14336, 100, ok, None) == IA
    assert lib.moe_ep_peer_plan(ok, ok, 4, 0, 256, ok, 14330, 100, ok, None) == IA
    assert lib.moe_ep_peer_plan(ok, ok, 4, 0, 256, ok, 14336, -1, ok, None) == IA
    assert lib.moe_ep_peer_plan(ok, ok, 4, 0, 256, None, 14336, 100, ok, None) == IA
    assert lib.moe_ep_peer_plan(ok, ok, 4, 0, 256, ok, 14336, 100, None, None) == IA
    # dispatch / collect / combine: pointers and alignment
    assert lib.moe_ep_peer_dispatch(ctypes.byref(c), None, ok, ok, 10, None) == IA
    assert lib.moe_ep_peer_dispatch(ctypes.byref(c), ok + 8, ok, ok, 10, None) == IA
    assert lib.moe_ep_peer_dispatch(ctypes.byref(c), ok, ok, None, 10, None) == IA
    assert lib.moe_ep_peer_dispatch(ctypes.byref(c), ok, ok, ok, -1, None) == IA
    assert lib.moe_ep_peer_dispatch(ctypes.byref(c), None, None, None, 0, None) == L.MOE_OK   # no rows
    assert lib.moe_ep_peer_collect(ctypes.byref(c), ok, ok, 10, ok + 8, None) == IA
    assert lib.moe_ep_peer_collect(ctypes.byref(c), None, ok, 10, ok, None) == IA
    assert lib.moe_ep_peer_collect(ctypes.byref(c), ok, None, 10, ok, None) == IA
    assert lib.moe_combine_peer(ctypes.byref(c), None, ok, ok, None, None, ok, None) == IA
    assert lib.moe_combine_peer(ctypes.byref(c), ok, ok, ok, None, None, ok + 4, None) == IA


def test_layer_rejects_unsupported_combinations():
    from dataclasses import replace
    w = synth.WORKLOADS["ec_deepseekmoe_16b"]
    with pytest.raises(ValueError):
        layer.MoELayer(replace(w, mxfp8=True), {}, "cpu")
    with pytest.raises(ValueError):
        layer.MoELayer(replace(synth.WORKLOADS["deepseek_v3"], fp8=True, f=1000), {}, "cpu")


def test_expert_parallel_layer_validation():
    from dataclasses import replace
    from sparse_mixture_experts_21_b200.ep import EPMoELayer
    w = synth.WORKLOADS["deepseek_v3"]
    with pytest.raises(ValueError):
        EPMoELayer(w, {}, 0, 3, "cpu")                       # 256 experts over 3 ranks
    with pytest.raises(ValueError):
        EPMoELayer(replace(w, mxfp8=True), {}, 0, 2, "cpu")  # the exchange carries bf16 rows
    with pytest.raises(ValueError):
        EPMoELayer(synth.WORKLOADS["ec_deepseekmoe_16b"], {}, 0, 2, "cpu")
    with pytest.raises(ValueError):
        EPMoELayer(w, {}, 0, 2, "cpu", peer=False, device_plan=True)   # the device plan needs peer memory


def test_capture_refuses_replica_mode():
    lay = layer.MoELayer(synth.WORKLOADS["tiny_top2_fp32"], {}, "cpu", group=object())
    with pytest.raises(ValueError):
        lay.capture(None)
