"""ctypes binding of the C ABI in include/moe_b200.h (argument marshalling only).

Every function here forwards torch tensors' device pointers and the current CUDA
stream to the library; all computation happens in the library's kernels.  There
is no fallback: if the shared library is missing, load() raises.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_double, c_float, c_int, c_int32, c_int64, c_size_t, c_void_p
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_NAME = "libmoe_b200.so"
LIB_PATH = os.path.join(_HERE, LIB_NAME)

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE_TOO_SMALL, MOE_ERR_CUDA, \
    MOE_ERR_DEVICE_TIMEOUT = range(6)
SCORE_SOFTMAX, SCORE_SIGMOID = 0, 1
DTYPE_F32, DTYPE_BF16 = 0, 1
CAP_DROPLESS, CAP_CEIL_CF_T_OVER_N, CAP_CF_K_T_OVER_N_FLOOR = 0, 1, 2

EXPORTED = ("moe_capacity", "moe_route_partials", "moe_workspace_size", "moe_route", "moe_permute",
            "moe_grouped_ffn", "moe_grouped_ffn_shared", "moe_grouped_ffn_gather", "moe_grouped_ffn_gate_up",
            "moe_grouped_ffn_down", "moe_combine", "moe_router_stats", "moe_bias_update",
            "moe_device_status", "moe_status_string", "moe_permute_noalloc", "moe_bias_update_ema",
            "moe_bias_update_seq", "moe_route_scores", "moe_expert_choice", "moe_combine_ec",
            "moe_selftest_wait_timeout", "moe_quantize_fp8", "moe_permute_fp8", "moe_grouped_ffn_fp8",
            "moe_quantize_mxfp8", "moe_permute_mxfp8", "moe_grouped_ffn_mxfp8", "moe_quantize_nvfp4",
            "moe_permute_nvfp4", "moe_grouped_ffn_nvfp4", "moe_ep_plan",
            "moe_rows_move", "moe_peer_export", "moe_peer_import", "moe_peer_close", "moe_ep_peer_plan",
            "moe_ep_peer_dispatch", "moe_ep_peer_collect", "moe_combine_peer", "moe_router_stats_partial", "moe_router_stats_finalize",
            "moe_expert_choice_capacity", "moe_route_prepare_size", "moe_route_prepare",
            "moe_last_cuda_error", "moe_last_cuda_error_string")

NEAR_TIE = 1e-4        # margin below which a token counts as a near-tie


class MoeConfig(ctypes.Structure):
    """Mirror of moe_config_t."""
    _fields_ = [("T", c_int64), ("d_model", c_int32), ("n_experts", c_int32), ("top_k", c_int32),
                ("d_ff", c_int32), ("score_fn", c_int32), ("renorm", c_int32), ("n_groups", c_int32),
                ("topk_groups", c_int32), ("group_score_topn", c_int32), ("capacity_mode", c_int32),
                ("x_dtype", c_int32), ("shared_sink", c_int32), ("capacity_factor", c_double)]


class MoeStats(ctypes.Structure):
    """Mirror of moe_stats_t."""
    _fields_ = [("aux", c_float), ("aux_raw", c_float), ("z", c_float), ("z_loss", c_float),
                ("cv", c_float), ("cv_kept", c_float), ("bias_norm", c_float), ("dead", c_int32),
                ("dropped_slots", c_int32), ("dropped_tokens", c_int32), ("R", c_int32),
                ("near_ties", c_int32), ("T", c_int64), ("reserved", c_int32 * 2)]


STATS_BYTES = ctypes.sizeof(MoeStats)


def stats_partial_len(n_experts: int) -> int:
    """Doubles in the sufficient-statistics vector (MOE_STATS_PARTIAL_LEN)."""
    return 3 * n_experts + 5


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn} failed: status {status} ({text})")
        self.status = status


_lib = None


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load the shared library (once).  Raises if it is absent."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise FileNotFoundError(
            f"{p} not found: build it with `python -m sparse_mixture_experts_21_b200.build`")
    lib = ctypes.CDLL(p)
    vp, i32p = c_void_p, POINTER(c_int32)
    cfgp = POINTER(MoeConfig)
    sig = {
        "moe_capacity": [cfgp, POINTER(c_int64)],
        "moe_route_partials": [cfgp, i32p],
        "moe_workspace_size": [cfgp, POINTER(c_size_t)],
        "moe_route": [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, c_size_t, vp],
        "moe_permute": [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, c_size_t, vp],
        "moe_permute_noalloc": [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp],
        "moe_grouped_ffn": [cfgp, vp, c_int64, vp, c_int32, vp, vp, vp, c_int32, vp, vp, vp],
        "moe_grouped_ffn_shared": [cfgp, vp, c_int64, vp, c_int32, vp, vp, vp, c_int32, vp, vp, vp, c_int64, vp, vp,
                                   vp, vp],
        "moe_grouped_ffn_gate_up": [cfgp, vp, c_int64, vp, c_int32, vp, vp, c_int32, vp, vp],
        "moe_grouped_ffn_down": [cfgp, vp, c_int64, vp, c_int32, vp, c_int32, vp, c_int64, vp, vp],
        "moe_grouped_ffn_gather": [cfgp, vp, c_int64, vp, c_int64, vp, c_int32, vp, vp, vp, c_int32, vp, vp, vp, vp,
                                   vp, vp],
        "moe_combine": [cfgp, vp, vp, vp, vp, vp, vp, vp],
        "moe_router_stats": [cfgp, vp, vp, vp, vp, vp, vp, c_float, vp, c_float, c_float, vp, vp, vp, vp],
        "moe_router_stats_partial": [cfgp, vp, vp, vp, vp, vp, vp, c_float, vp, vp],
        "moe_router_stats_finalize": [cfgp, vp, vp, c_float, c_float, vp, vp, vp, vp, vp],
        "moe_expert_choice_capacity": [cfgp, i32p],
        "moe_route_prepare_size": [cfgp, POINTER(c_size_t)],
        "moe_route_prepare": [cfgp, vp, vp, c_size_t, vp],
        "moe_bias_update": [cfgp, vp, vp, c_float, c_float, vp],
        "moe_bias_update_ema": [cfgp, vp, vp, c_float, vp, c_float, c_float, vp],
        "moe_bias_update_seq": [cfgp, vp, vp, c_int32, vp, c_float, c_float, vp, c_size_t, vp],
        "moe_route_scores": [cfgp, vp, vp, vp, vp, vp, vp, vp, c_size_t, vp],
        "moe_expert_choice": [cfgp, vp, vp, c_int32, vp, vp, vp, vp, vp, vp],
        "moe_combine_ec": [cfgp, vp, vp, vp, vp, vp, vp, vp],
        "moe_device_status": [i32p, c_int32],
        "moe_selftest_wait_timeout": [c_int64, vp, vp],
        "moe_status_string": [c_int],
        "moe_last_cuda_error": [],
        "moe_last_cuda_error_string": [],
        "moe_quantize_fp8": [vp, c_int64, c_int32, c_int32, vp, vp, vp],
        "moe_permute_fp8": [cfgp, vp, vp, vp, vp, vp, vp, vp],
        "moe_grouped_ffn_fp8": [cfgp, vp, vp, c_int64, vp, c_int32, vp, vp, vp, vp, vp, vp, c_int32, vp, vp,
                                vp, vp],
        "moe_quantize_mxfp8": [vp, c_int64, c_int32, vp, vp, vp],
        "moe_ep_plan": [vp, c_int32, c_int32, c_int32, vp, vp, vp, vp, c_int64, vp],
        "moe_rows_move": [vp, c_int64, vp, vp, c_int64, c_int32, vp, vp],
        "moe_peer_export": [vp, vp],
        "moe_peer_import": [vp, ctypes.POINTER(vp)],
        "moe_peer_close": [vp],
        "moe_ep_peer_plan": [vp, vp, c_int32, c_int32, c_int32, vp, c_int64, c_int64, vp, vp],
        "moe_ep_peer_dispatch": [cfgp, vp, vp, vp, c_int64, vp],
        "moe_ep_peer_collect": [cfgp, vp, vp, c_int64, vp, vp],
        "moe_combine_peer": [cfgp, vp, vp, vp, vp, vp, vp, vp],
        "moe_permute_mxfp8": [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp],
        "moe_grouped_ffn_mxfp8": [cfgp, vp, vp, c_int64, vp, c_int32, vp, vp, vp, vp, vp, vp, c_int32, vp, vp,
                                  vp, vp],
        "moe_quantize_nvfp4": [vp, c_int64, c_int32, c_int32, vp, vp, vp, vp],
        "moe_permute_nvfp4": [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp],
        "moe_grouped_ffn_nvfp4": [cfgp, vp, vp, c_int64, vp, c_int32, vp, vp, vp, vp, vp, vp, vp, vp, vp, c_int32,
                                  vp, vp, vp, vp],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = c_char_p if name in ("moe_status_string", "moe_last_cuda_error_string") else c_int
    if path is None:
        _lib = lib
    return lib


# ----------------------------------------------------------------------------- helpers
def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the MoE library must be contiguous")
    return t.data_ptr()


def _stream(stream=None) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check(name: str, status: int) -> None:
    if status != MOE_OK:
        text = load().moe_status_string(status).decode()
        if status == MOE_ERR_CUDA:
            text += ": " + load().moe_last_cuda_error_string().decode()
        raise MoeError(name, status, text)


def capacity(cfg: MoeConfig) -> int:
    out = c_int64()
    _check("moe_capacity", load().moe_capacity(ctypes.byref(cfg), ctypes.byref(out)))
    return out.value


def route_partials(cfg: MoeConfig) -> int:
    out = c_int32()
    _check("moe_route_partials", load().moe_route_partials(ctypes.byref(cfg), ctypes.byref(out)))
    return out.value


def workspace_size(cfg: MoeConfig) -> int:
    out = c_size_t()
    _check("moe_workspace_size", load().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(out)))
    return out.value


# ----------------------------------------------------------------------------- entry points
def moe_route(cfg, x, w_gate, logit_offset, bias, topk_idx, topk_w, lse, p_partial, margin, ws,
              stream=None, shared_w=None):
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("moe_route", load().moe_route(
        ctypes.byref(cfg), _ptr(x), _ptr(w_gate), _ptr(logit_offset), _ptr(bias), _ptr(topk_idx),
        _ptr(topk_w), _ptr(lse), _ptr(p_partial), _ptr(margin), _ptr(shared_w), _ptr(ws), nbytes,
        _stream(stream)))


def route_prepare_size(cfg: MoeConfig) -> int:
    out = c_size_t()
    _check("moe_route_prepare_size", load().moe_route_prepare_size(ctypes.byref(cfg), ctypes.byref(out)))
    return out.value


def moe_route_prepare(cfg, w_gate, prepared, stream=None):
    """Write the router weight's exact bf16 split into `prepared` (a uint8 tensor)."""
    _check("moe_route_prepare", load().moe_route_prepare(
        ctypes.byref(cfg), _ptr(w_gate), _ptr(prepared), prepared.numel() * prepared.element_size(),
        _stream(stream)))


def moe_permute(cfg, x, topk_idx, counts, offsets, row_of_slot, token_of_row, x_perm, n_dropped,
                ws, stream=None):
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("moe_permute", load().moe_permute(
        ctypes.byref(cfg), _ptr(x), _ptr(topk_idx), _ptr(counts), _ptr(offsets), _ptr(row_of_slot),
        _ptr(token_of_row), _ptr(x_perm), _ptr(n_dropped), _ptr(ws), nbytes, _stream(stream)))


def moe_permute_noalloc(cfg, x, topk_idx, counts, offsets, row_of_slot, token_of_row, x_perm,
                        n_dropped, stream=None):
    """moe_permute without a workspace (scratch kept inside the library)."""
    _check("moe_permute_noalloc", load().moe_permute_noalloc(
        ctypes.byref(cfg), _ptr(x), _ptr(topk_idx), _ptr(counts), _ptr(offsets), _ptr(row_of_slot),
        _ptr(token_of_row), _ptr(x_perm), _ptr(n_dropped), _stream(stream)))


def moe_grouped_ffn(cfg, x_rows, rows_cap, offsets, G, w1, w3, w2, f, h_scratch, y_rows, stream=None):
    _check("moe_grouped_ffn", load().moe_grouped_ffn(
        ctypes.byref(cfg), _ptr(x_rows), int(rows_cap), _ptr(offsets), int(G), _ptr(w1), _ptr(w3),
        _ptr(w2), int(f), _ptr(h_scratch), _ptr(y_rows), _stream(stream)))


def moe_grouped_ffn_shared(cfg, x_rows, rows_cap, offsets, G, w1, w3, w2, f, h_scratch, y_rows, x, T, ws1, ws3,
                           ws2, stream=None):
    """moe_grouped_ffn plus the shared expert (one dense group over x, its rows after
    the routed rows_cap rows of h_scratch and y_rows) in the same launches."""
    _check("moe_grouped_ffn_shared", load().moe_grouped_ffn_shared(
        ctypes.byref(cfg), _ptr(x_rows), int(rows_cap), _ptr(offsets), int(G), _ptr(w1), _ptr(w3), _ptr(w2), int(f),
        _ptr(h_scratch), _ptr(y_rows), _ptr(x), int(T), _ptr(ws1), _ptr(ws3), _ptr(ws2), _stream(stream)))


def moe_grouped_ffn_gate_up(cfg, x_rows, rows_cap, offsets, G, w1, w3, f, h_rows, stream=None):
    """The first pass of moe_grouped_ffn alone (bf16): h = silu(x W1^T) * (x W3^T) per group."""
    _check("moe_grouped_ffn_gate_up", load().moe_grouped_ffn_gate_up(
        ctypes.byref(cfg), _ptr(x_rows), int(rows_cap), _ptr(offsets), int(G), _ptr(w1), _ptr(w3), int(f),
        _ptr(h_rows), _stream(stream)))


def moe_grouped_ffn_down(cfg, h_rows, rows_cap, offsets, G, w2, f, y_rows, T=0, ws2=None, stream=None):
    """The second pass alone (bf16): y = h W2^T per group; with T and ws2, also the shared
    expert's T rows after rows_cap through ws2, in the same launch."""
    _check("moe_grouped_ffn_down", load().moe_grouped_ffn_down(
        ctypes.byref(cfg), _ptr(h_rows), int(rows_cap), _ptr(offsets), int(G), _ptr(w2), int(f), _ptr(y_rows),
        int(T), _ptr(ws2), _stream(stream)))


def moe_grouped_ffn_gather(cfg, x, T, token_of_row, rows_cap, offsets, G, w1, w3, w2, f, h_scratch, y_rows,
                           stream=None, ws1=None, ws3=None, ws2=None):
    """moe_grouped_ffn with row r read from x[token_of_row[r]] (bf16 only); with ws1, ws3,
    ws2 the shared expert over x rides in the same launches (its rows after rows_cap)."""
    _check("moe_grouped_ffn_gather", load().moe_grouped_ffn_gather(
        ctypes.byref(cfg), _ptr(x), int(T), _ptr(token_of_row), int(rows_cap), _ptr(offsets), int(G), _ptr(w1),
        _ptr(w3), _ptr(w2), int(f), _ptr(h_scratch), _ptr(y_rows), _ptr(ws1), _ptr(ws3), _ptr(ws2),
        _stream(stream)))


def moe_quantize_fp8(x, block_rows, q, scales, stream=None):
    """Block-quantise a bf16 matrix [rows, cols] to E4M3 codes (uint8) and fp32 scales."""
    rows, cols = x.shape
    _check("moe_quantize_fp8", load().moe_quantize_fp8(
        _ptr(x), int(rows), int(cols), int(block_rows), _ptr(q), _ptr(scales), _stream(stream)))


def moe_permute_fp8(cfg, x, row_of_slot, xq_perm, xs_perm, xq=None, xs=None, stream=None):
    _check("moe_permute_fp8", load().moe_permute_fp8(
        ctypes.byref(cfg), _ptr(x), _ptr(row_of_slot), _ptr(xq_perm), _ptr(xs_perm), _ptr(xq), _ptr(xs),
        _stream(stream)))


def moe_grouped_ffn_fp8(cfg, xq_rows, xs_rows, rows_cap, offsets, G, w1q, w1s, w3q, w3s, w2q, w2s, f,
                        hq_scratch, hs_scratch, y_rows, stream=None):
    _check("moe_grouped_ffn_fp8", load().moe_grouped_ffn_fp8(
        ctypes.byref(cfg), _ptr(xq_rows), _ptr(xs_rows), int(rows_cap), _ptr(offsets), int(G), _ptr(w1q),
        _ptr(w1s), _ptr(w3q), _ptr(w3s), _ptr(w2q), _ptr(w2s), int(f), _ptr(hq_scratch), _ptr(hs_scratch),
        _ptr(y_rows), _stream(stream)))


def mx_scales(rows: int, cols: int, device, groups: int = 0) -> torch.Tensor:
    """Buffer for MXFP8 scales in tile-atom order: rows cut into 128-row tiles (per group
    when `groups` > 0), one 512-byte atom per (tile, 128-wide K block)."""
    tiles = (rows + 127) // 128 + groups
    return torch.empty(max(tiles, 1) * (cols // 128) * 512, dtype=torch.uint8, device=device)


def moe_quantize_mxfp8(x, q, sf, stream=None):
    """MXFP8-quantise a bf16 matrix [rows, cols] along its rows: E4M3 codes and E8M0 scales
    (sf from mx_scales(rows, cols))."""
    rows, cols = x.shape
    _check("moe_quantize_mxfp8", load().moe_quantize_mxfp8(
        _ptr(x), int(rows), int(cols), _ptr(q), _ptr(sf), _stream(stream)))


def moe_permute_mxfp8(cfg, x, topk_idx, row_of_slot, offsets, q_perm, sf_perm, q=None, sf=None, stream=None):
    _check("moe_permute_mxfp8", load().moe_permute_mxfp8(
        ctypes.byref(cfg), _ptr(x), _ptr(topk_idx), _ptr(row_of_slot), _ptr(offsets), _ptr(q_perm),
        _ptr(sf_perm), _ptr(q), _ptr(sf), _stream(stream)))


def moe_grouped_ffn_mxfp8(cfg, xq_rows, xsf_rows, rows_cap, offsets, G, w1q, w1sf, w3q, w3sf, w2q, w2sf, f,
                          hq_scratch, hsf_scratch, y_rows, stream=None):
    _check("moe_grouped_ffn_mxfp8", load().moe_grouped_ffn_mxfp8(
        ctypes.byref(cfg), _ptr(xq_rows), _ptr(xsf_rows), int(rows_cap), _ptr(offsets), int(G), _ptr(w1q),
        _ptr(w1sf), _ptr(w3q), _ptr(w3sf), _ptr(w2q), _ptr(w2sf), int(f), _ptr(hq_scratch), _ptr(hsf_scratch),
        _ptr(y_rows), _stream(stream)))


def nv_scales(rows: int, cols: int, device, groups: int = 0) -> torch.Tensor:
    """Buffer for NVFP4 scales in tile-atom order: rows cut into 128-row tiles (per group
    when `groups` > 0), one 512-byte atom per (tile, 64-wide K chunk)."""
    tiles = (rows + 127) // 128 + groups
    return torch.empty(max(tiles, 1) * (cols // 64) * 512, dtype=torch.uint8, device=device)


def moe_quantize_nvfp4(x, q, sf, g=None, tensor_rows=0, stream=None):
    """NVFP4-quantise a bf16 matrix [rows, cols] along its rows: packed E2M1 codes
    (q: rows x cols / 2 bytes), E4M3 block scales (sf from nv_scales(rows, cols)) and,
    with tensor_rows > 0, one tensor scale per tensor_rows rows into g."""
    rows, cols = x.shape
    _check("moe_quantize_nvfp4", load().moe_quantize_nvfp4(
        _ptr(x), int(rows), int(cols), int(tensor_rows), _ptr(q), _ptr(sf), _ptr(g), _stream(stream)))


def moe_permute_nvfp4(cfg, x, topk_idx, row_of_slot, offsets, q_perm, sf_perm, q=None, sf=None, stream=None):
    _check("moe_permute_nvfp4", load().moe_permute_nvfp4(
        ctypes.byref(cfg), _ptr(x), _ptr(topk_idx), _ptr(row_of_slot), _ptr(offsets), _ptr(q_perm),
        _ptr(sf_perm), _ptr(q), _ptr(sf), _stream(stream)))


def moe_grouped_ffn_nvfp4(cfg, xq_rows, xsf_rows, rows_cap, offsets, G, w1q, w1sf, g1, w3q, w3sf, g3, w2q, w2sf,
                          g2, f, hq_scratch, hsf_scratch, y_rows, stream=None):
    _check("moe_grouped_ffn_nvfp4", load().moe_grouped_ffn_nvfp4(
        ctypes.byref(cfg), _ptr(xq_rows), _ptr(xsf_rows), int(rows_cap), _ptr(offsets), int(G), _ptr(w1q),
        _ptr(w1sf), _ptr(g1), _ptr(w3q), _ptr(w3sf), _ptr(g3), _ptr(w2q), _ptr(w2sf), _ptr(g2), int(f),
        _ptr(hq_scratch), _ptr(hsf_scratch), _ptr(y_rows), _stream(stream)))


def moe_ep_plan(offsets_all, world, rank, send_splits, recv_splits, local_offsets, regroup_map, stream=None):
    """Split sizes, local expert offsets and the regroup map of one rank (offsets_all [W, N + 1])."""
    _check("moe_ep_plan", load().moe_ep_plan(
        _ptr(offsets_all), int(world), int(rank), int(offsets_all.shape[1]) - 1, _ptr(send_splits), _ptr(recv_splits),
        _ptr(local_offsets), _ptr(regroup_map), int(regroup_map.shape[0]), _stream(stream)))


def moe_rows_move(src, map_, n_rows, dst, scatter=False, rows_cap=None, stream=None):
    """dst[r] = src[map[r]] (gather) or dst[map[r]] = src[r] (scatter) for r < n_rows
    (a device int32 scalar, or None for rows_cap = len(map))."""
    row_bytes = src.stride(0) * src.element_size()
    _check("moe_rows_move", load().moe_rows_move(
        _ptr(src), int(row_bytes), _ptr(map_), _ptr(n_rows), int(map_.shape[0] if rows_cap is None else rows_cap),
        1 if scatter else 0, _ptr(dst), _stream(stream)))


PEER_HANDLE_BYTES = 72


def moe_peer_export(t: torch.Tensor) -> bytes:
    """Handle (CUDA IPC handle of t's allocation + t's offset in it) for other processes."""
    buf = ctypes.create_string_buffer(PEER_HANDLE_BYTES)
    _check("moe_peer_export", load().moe_peer_export(_ptr(t), buf))
    return buf.raw


def moe_peer_import(handle: bytes) -> int:
    """Device address of another process's exported buffer (until moe_peer_close)."""
    if len(handle) != PEER_HANDLE_BYTES:
        raise ValueError(f"a peer handle has {PEER_HANDLE_BYTES} bytes, not {len(handle)}")
    out = ctypes.c_void_p()
    _check("moe_peer_import", load().moe_peer_import(ctypes.create_string_buffer(handle, len(handle)),
                                                     ctypes.byref(out)))
    return int(out.value)


def moe_peer_close(ptr: int) -> None:
    _check("moe_peer_close", load().moe_peer_close(ctypes.c_void_p(ptr)))


def moe_ep_peer_plan(offsets_round, offsets_own, world, rank, peer_rows, row_bytes, recv_cap, row_addr, stream=None):
    """row_addr[i]: where row i of this rank lands in its expert's rank's receive buffer
    this round (0 outside the round).  peer_rows: uint64/int64 [W] device addresses."""
    _check("moe_ep_peer_plan", load().moe_ep_peer_plan(
        _ptr(offsets_round), _ptr(offsets_own), int(world), int(rank), int(offsets_own.shape[0]) - 1, _ptr(peer_rows),
        int(row_bytes), int(recv_cap), _ptr(row_addr), _stream(stream)))


def moe_ep_peer_dispatch(cfg, x, row_of_slot, row_addr, rows_cap=None, stream=None):
    """*row_addr[row_of_slot[t, j]] = x[t] for the slots of this round (the permutation's
    gather and the dispatch in one pass)."""
    _check("moe_ep_peer_dispatch", load().moe_ep_peer_dispatch(
        ctypes.byref(cfg), _ptr(x), _ptr(row_of_slot), _ptr(row_addr),
        int(row_addr.shape[0] if rows_cap is None else rows_cap), _stream(stream)))


def moe_ep_peer_collect(cfg, row_addr, n_rows, y_perm, rows_cap=None, stream=None):
    """y_perm[i] = *row_addr[i] for the rows of this round."""
    _check("moe_ep_peer_collect", load().moe_ep_peer_collect(
        ctypes.byref(cfg), _ptr(row_addr), _ptr(n_rows), int(row_addr.shape[0] if rows_cap is None else rows_cap),
        _ptr(y_perm), _stream(stream)))


def moe_combine_peer(cfg, row_addr, row_of_slot, topk_w, shared_out, y, stream=None, shared_w=None):
    """moe_combine reading the result of row r at row_addr[r]."""
    _check("moe_combine_peer", load().moe_combine_peer(
        ctypes.byref(cfg), _ptr(row_addr), _ptr(row_of_slot), _ptr(topk_w), _ptr(shared_out), _ptr(shared_w),
        _ptr(y), _stream(stream)))


def moe_combine(cfg, y_perm, row_of_slot, topk_w, shared_out, y, stream=None, shared_w=None):
    _check("moe_combine", load().moe_combine(
        ctypes.byref(cfg), _ptr(y_perm), _ptr(row_of_slot), _ptr(topk_w), _ptr(shared_out),
        _ptr(shared_w), _ptr(y), _stream(stream)))


def moe_router_stats(cfg, counts, offsets, p_partial, lse, n_dropped, bias, alpha, z_coef, stats,
                     f_out=None, p_out=None, stream=None, margin=None, near_tie=NEAR_TIE):
    _check("moe_router_stats", load().moe_router_stats(
        ctypes.byref(cfg), _ptr(counts), _ptr(offsets), _ptr(p_partial), _ptr(lse), _ptr(n_dropped),
        _ptr(margin), float(near_tie), _ptr(bias), float(alpha), float(z_coef), _ptr(stats), _ptr(f_out),
        _ptr(p_out), _stream(stream)))


def moe_router_stats_partial(cfg, counts, offsets, p_partial, lse, n_dropped, partial, margin=None,
                             near_tie=NEAR_TIE, stream=None):
    """This batch's sufficient statistics (fp64 [3N + 5]) for a sum over ranks."""
    _check("moe_router_stats_partial", load().moe_router_stats_partial(
        ctypes.byref(cfg), _ptr(counts), _ptr(offsets), _ptr(p_partial), _ptr(lse), _ptr(n_dropped),
        _ptr(margin), float(near_tie), _ptr(partial), _stream(stream)))


def moe_router_stats_finalize(cfg, partial, bias, alpha, z_coef, stats, f_out=None, p_out=None,
                              counts_out=None, stream=None):
    """Statistics of the (summed) sufficient-statistics vector."""
    _check("moe_router_stats_finalize", load().moe_router_stats_finalize(
        ctypes.byref(cfg), _ptr(partial), _ptr(bias), float(alpha), float(z_coef), _ptr(stats), _ptr(f_out),
        _ptr(p_out), _ptr(counts_out), _stream(stream)))


def moe_bias_update(cfg, counts, bias, rate, clamp=0.0, stream=None):
    _check("moe_bias_update", load().moe_bias_update(
        ctypes.byref(cfg), _ptr(counts), _ptr(bias), float(rate), float(clamp), _stream(stream)))


def moe_bias_update_ema(cfg, counts, ema, beta, bias, rate, clamp=0.0, stream=None):
    _check("moe_bias_update_ema", load().moe_bias_update_ema(
        ctypes.byref(cfg), _ptr(counts), _ptr(ema), float(beta), _ptr(bias), float(rate), float(clamp),
        _stream(stream)))


def moe_bias_update_seq(cfg, topk_idx, seq_offsets, n_seq, bias, rate, clamp, ws, stream=None):
    nbytes = ws.numel() * ws.element_size()
    _check("moe_bias_update_seq", load().moe_bias_update_seq(
        ctypes.byref(cfg), _ptr(topk_idx), _ptr(seq_offsets), int(n_seq), _ptr(bias), float(rate),
        float(clamp), _ptr(ws), nbytes, _stream(stream)))


def moe_route_scores(cfg, x, w_gate, logit_offset, scores, lse, p_partial, ws, stream=None):
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("moe_route_scores", load().moe_route_scores(
        ctypes.byref(cfg), _ptr(x), _ptr(w_gate), _ptr(logit_offset), _ptr(scores), _ptr(lse),
        _ptr(p_partial), _ptr(ws), nbytes, _stream(stream)))


def expert_choice_capacity(cfg: MoeConfig) -> int:
    """Expert-choice capacity C = min(T, ceil(cf k T / N)) computed by the library."""
    out = c_int32()
    _check("moe_expert_choice_capacity", load().moe_expert_choice_capacity(ctypes.byref(cfg), ctypes.byref(out)))
    return out.value


def moe_expert_choice(cfg, x, scores, capacity, row_of, token_of_row, offsets, x_perm, n_unpicked=None,
                      stream=None):
    _check("moe_expert_choice", load().moe_expert_choice(
        ctypes.byref(cfg), _ptr(x), _ptr(scores), int(capacity), _ptr(row_of), _ptr(token_of_row),
        _ptr(offsets), _ptr(x_perm), _ptr(n_unpicked), _stream(stream)))


def moe_combine_ec(cfg, y_perm, row_of, scores, shared_out, y, n_unpicked=None, stream=None):
    _check("moe_combine_ec", load().moe_combine_ec(
        ctypes.byref(cfg), _ptr(y_perm), _ptr(row_of), _ptr(scores), _ptr(shared_out), _ptr(y),
        _ptr(n_unpicked), _stream(stream)))


def moe_selftest_wait_timeout(limit_cycles, completed=None, stream=None):
    _check("moe_selftest_wait_timeout", load().moe_selftest_wait_timeout(
        int(limit_cycles), _ptr(completed), _stream(stream)))


def moe_device_status(reset: bool = True) -> int:
    out = c_int32()
    _check("moe_device_status", load().moe_device_status(ctypes.byref(out), 1 if reset else 0))
    return out.value


def stats_from_tensor(t: torch.Tensor) -> dict:
    """Decode a moe_stats_t held in a uint8 tensor of STATS_BYTES."""
    raw = bytes(t.detach().cpu().numpy().tobytes())
    s = MoeStats.from_buffer_copy(raw)
    return {name: getattr(s, name) for name, _ in MoeStats._fields_ if name != "reserved"}
