"""ctypes binding of the C ABI in include/moe_mxfp8.h.

Argument marshalling only: every function here has the name and the
arguments of its C counterpart (device pointers as Python ints, sizes as
ints, streams as raw cudaStream_t handles) and raises MoeError on a non-zero
status.  All computation happens in the CUDA library; if the library is
missing this module raises at import time instead of falling back to any
other implementation.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_mxfp8.so")

MOE_QUANT_ROW = 1
MOE_QUANT_COL = 2
MOE_OP_PERMUTE = 1
MOE_OP_FWD = 2
MOE_OP_BWD = 3
MOE_OP_FWD_BF16 = 4
MOE_OP_FWD_FP8_TENSOR = 5
MOE_OP_BWD_BF16 = 6
MOE_OP_BWD_FP8_TENSOR = 7
MOE_MAX_EXPERTS = 256

STATUS = {
    0: "MOE_OK", 1: "MOE_ERR_INVALID", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
    4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_INDEX", 6: "MOE_ERR_TIMEOUT", 7: "MOE_ERR_NO_DEVICE",
    8: "MOE_ERR_TOO_LARGE",
}
MOE_PERMUTE_NOALLOC_SCRATCH_BYTES = 256 * 1024

EXPORTED = [
    "moe_mx_scale_bytes", "moe_padded_rows", "moe_workspace_size", "moe_mlp_quantize_mxfp8",
    "moe_permute", "moe_grouped_mlp_fwd", "moe_combine", "moe_grouped_mlp_bwd",
    "moe_get_device_status", "moe_status_string", "moe_launch_count", "moe_selftest_wait_timeout",
    "moe_timing_enable", "moe_timing_read", "moe_permute_noalloc", "moe_mlp_quantize_weights",
    "moe_router_topk", "moe_mx_scales_to_blocked", "moe_mx_scales_from_blocked", "moe_route_permute",
    "moe_grouped_mlp_fwd_bf16", "moe_grouped_mlp_fwd_fp8_tensor", "moe_grouped_mlp_bwd_bf16",
    "moe_grouped_mlp_bwd_fp8_tensor",
]
MOE_DTYPE_F32, MOE_DTYPE_BF16 = 0, 1


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} ({status_string(code)})")


if not os.path.exists(LIB_PATH):
    raise ImportError(f"CUDA library not built: {LIB_PATH} (run python -m "
                      "mxfp8_grouped_gemm_x32_b200.build_lib)")
_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t


def _decl(name, res, *args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_decl("moe_mx_scale_bytes", _I64, _I32, _I64, _I64)
_decl("moe_padded_rows", _I64, _I32, _I32, _I32)
_decl("moe_workspace_size", _I64, _I32, _I32, _I32, _I32, _I32, _I32)
_decl("moe_mlp_quantize_mxfp8", _I32, _P, _I32, _I64, _I64, _I32, _P, _P, _P)
_decl("moe_mlp_quantize_weights", _I32, _P, _P, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _P)
_decl("moe_permute", _I32, _P, _P, _P, _I32, _I32, _I32, _I32, _I64, _P, _P, _P, _P, _P, _P, _P, _P,
      _P, _P, _SZ, _P)
_decl("moe_grouped_mlp_fwd", _I32, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I64, _P, _P, _P,
      _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P)
_decl("moe_combine", _I32, _P, _I32, _I32, _I32, _P, _P)
_decl("moe_router_topk", _I32, _P, _I32, _I32, _I32, _I32, _P, _P, _P)
_decl("moe_grouped_mlp_bwd", _I32, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I64, _P, _P, _P,
      _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P)
_decl("moe_mx_scales_to_blocked", _I32, _P, _I32, _I64, _I64, _I64, _P, _P)
_decl("moe_mx_scales_from_blocked", _I32, _P, _I32, _I64, _I64, _P, _I64, _P)
_decl("moe_route_permute", _I32, _P, _I32, _P, _I32, _I32, _I32, _I32, _I64, _P, _P, _P, _P, _P, _P, _P, _P,
      _P, _P, _P, _P, _SZ, _P)
_decl("moe_grouped_mlp_fwd_bf16", _I32, _P, _P, _I32, _I32, _I32, _I32, _I32, _I64, _P, _P, _P, _P, _P, _P, _P,
      _P, _P, _SZ, _P)
_decl("moe_grouped_mlp_bwd_bf16", _I32, _P, _P, _I32, _I32, _I32, _I32, _I32, _I64, _P, _P, _P, _P, _P, _P,
      _P, _P, _P, _P, _P, _P, _P, _SZ, _P)
_decl("moe_grouped_mlp_fwd_fp8_tensor", _I32, _P, _P, _I32, _I32, _I32, _I32, _I32, _I64, _P, _P, _P, _P, _P, _P,
      _P, _P, _P, _P, _SZ, _P)
_decl("moe_grouped_mlp_bwd_fp8_tensor", _I32, _P, _P, _I32, _I32, _I32, _I32, _I32, _I64, _P, _P, _P, _P, _P, _P,
      _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P)
_decl("moe_get_device_status", _I32, _P)
_decl("moe_status_string", ctypes.c_char_p, _I32)
_decl("moe_launch_count", _I64, _I32)
_decl("moe_selftest_wait_timeout", _I32, _I32, _P)
_decl("moe_permute_noalloc", _I32, _P, _P, _P, _I32, _I32, _I32, _I32, _I64, _P, _P, _P, _P, _P, _P,
      _P, _P, _P, _P)
_decl("moe_timing_enable", _I32, _I32)
_decl("moe_timing_read", _I32, ctypes.c_char_p, _I64, ctypes.POINTER(ctypes.c_double),
      ctypes.POINTER(_I64), _I32)


def _check(fn: str, code: int) -> None:
    if code != 0:
        raise MoeError(fn, code)


def status_string(code: int) -> str:
    return _lib.moe_status_string(code).decode()


def moe_mx_scale_bytes(groups: int, rows: int, k: int) -> int:
    return _lib.moe_mx_scale_bytes(groups, rows, k)


def moe_padded_rows(T: int, k: int, E: int) -> int:
    return _lib.moe_padded_rows(T, k, E)


def moe_workspace_size(op: int, T: int, k: int, E: int, H: int, I: int) -> int:
    return _lib.moe_workspace_size(op, T, k, E, H, I)


def moe_mlp_quantize_mxfp8(src, groups, rows, cols, mode, q, sf, stream=0):
    _check("moe_mlp_quantize_mxfp8", _lib.moe_mlp_quantize_mxfp8(src, groups, rows, cols, mode, q, sf, stream))


def moe_mlp_quantize_weights(w_gate_up, w_down, E, H, I, w1q, w1sf, w2q, w2sf, w1tq, w1tsf, w2tq, w2tsf,
                             stream=0):
    _check("moe_mlp_quantize_weights", _lib.moe_mlp_quantize_weights(
        w_gate_up, w_down, E, H, I, w1q, w1sf, w2q, w2sf, w1tq, w1tsf, w2tq, w2tsf, stream))


def moe_permute(x, topk_idx, topk_prob, T, H, k, E, rows_cap, split_sizes, group_offsets, row_to_slot,
                slot_to_row, prob_perm, xq, xq_sf, xq_col, xq_col_sf, workspace, workspace_bytes, stream=0):
    _check("moe_permute", _lib.moe_permute(x, topk_idx, topk_prob, T, H, k, E, rows_cap, split_sizes,
                                           group_offsets, row_to_slot, slot_to_row, prob_perm, xq, xq_sf,
                                           xq_col, xq_col_sf, workspace, workspace_bytes, stream))


def moe_permute_noalloc(x, topk_idx, topk_prob, T, H, k, E, rows_cap, split_sizes, group_offsets,
                        row_to_slot, slot_to_row, prob_perm, xq, xq_sf, xq_col, xq_col_sf, stream=0):
    """moe_permute for callers that cannot provide a device workspace: the
    scratch lives in the library's built-in device array (see the header)."""
    _check("moe_permute_noalloc", _lib.moe_permute_noalloc(
        x, topk_idx, topk_prob, T, H, k, E, rows_cap, split_sizes, group_offsets, row_to_slot,
        slot_to_row, prob_perm, xq, xq_sf, xq_col, xq_col_sf, stream))


def moe_grouped_mlp_fwd(w1q, w1sf, w2q, w2sf, T, H, I, E, k, rows_cap, split_sizes, group_offsets,
                        row_to_slot, slot_to_row, prob_perm, xq, xq_sf, out, saved_a, hq, hq_sf, workspace,
                        workspace_bytes, stream=0):
    _check("moe_grouped_mlp_fwd", _lib.moe_grouped_mlp_fwd(
        w1q, w1sf, w2q, w2sf, T, H, I, E, k, rows_cap, split_sizes, group_offsets, row_to_slot, slot_to_row,
        prob_perm, xq, xq_sf, out, saved_a, hq, hq_sf, workspace, workspace_bytes, stream))


def moe_mx_scales_to_blocked(plain, groups, rows, k, ld, blocked, stream=0):
    _check("moe_mx_scales_to_blocked", _lib.moe_mx_scales_to_blocked(plain, groups, rows, k, ld, blocked, stream))


def moe_mx_scales_from_blocked(blocked, groups, rows, k, plain, ld, stream=0):
    _check("moe_mx_scales_from_blocked", _lib.moe_mx_scales_from_blocked(blocked, groups, rows, k, plain, ld, stream))


def moe_grouped_mlp_fwd_bf16(w_gate_up, w_down, T, H, I, E, k, rows_cap, split_sizes, group_offsets, row_to_slot,
                             slot_to_row, prob_perm, x, out, saved_a, workspace, workspace_bytes, stream=0):
    _check("moe_grouped_mlp_fwd_bf16", _lib.moe_grouped_mlp_fwd_bf16(
        w_gate_up, w_down, T, H, I, E, k, rows_cap, split_sizes, group_offsets, row_to_slot, slot_to_row, prob_perm,
        x, out, saved_a, workspace, workspace_bytes, stream))


def moe_grouped_mlp_bwd_bf16(w_gate_up, w_down, T, H, I, E, k, rows_cap, split_sizes, group_offsets, row_to_slot,
                             slot_to_row, prob_perm, dY, saved_a, x, dX, dW1, dW2, dprob, workspace,
                             workspace_bytes, stream=0):
    _check("moe_grouped_mlp_bwd_bf16", _lib.moe_grouped_mlp_bwd_bf16(
        w_gate_up, w_down, T, H, I, E, k, rows_cap, split_sizes, group_offsets, row_to_slot, slot_to_row, prob_perm,
        dY, saved_a, x, dX, dW1, dW2, dprob, workspace, workspace_bytes, stream))


def moe_grouped_mlp_fwd_fp8_tensor(w_gate_up, w_down, T, H, I, E, k, rows_cap, split_sizes, group_offsets,
                                   row_to_slot, slot_to_row, prob_perm, x, out, saved_a, scales, workspace,
                                   workspace_bytes, stream=0):
    _check("moe_grouped_mlp_fwd_fp8_tensor", _lib.moe_grouped_mlp_fwd_fp8_tensor(
        w_gate_up, w_down, T, H, I, E, k, rows_cap, split_sizes, group_offsets, row_to_slot, slot_to_row, prob_perm,
        x, out, saved_a, scales, workspace, workspace_bytes, stream))


def moe_grouped_mlp_bwd_fp8_tensor(w_gate_up, w_down, T, H, I, E, k, rows_cap, split_sizes, group_offsets,
                                   row_to_slot, slot_to_row, prob_perm, dY, saved_a, x, fwd_scales, dX, dW1, dW2,
                                   dprob, scales, workspace, workspace_bytes, stream=0):
    _check("moe_grouped_mlp_bwd_fp8_tensor", _lib.moe_grouped_mlp_bwd_fp8_tensor(
        w_gate_up, w_down, T, H, I, E, k, rows_cap, split_sizes, group_offsets, row_to_slot, slot_to_row, prob_perm,
        dY, saved_a, x, fwd_scales, dX, dW1, dW2, dprob, scales, workspace, workspace_bytes, stream))


def moe_combine(y, T, k, H, out, stream=0):
    _check("moe_combine", _lib.moe_combine(y, T, k, H, out, stream))


def moe_router_topk(logits, logits_dtype, T, E, k, topk_idx, topk_prob, stream=0):
    _check("moe_router_topk", _lib.moe_router_topk(logits, logits_dtype, T, E, k, topk_idx, topk_prob, stream))


def moe_route_permute(logits, logits_dtype, x, T, H, k, E, rows_cap, topk_idx, topk_prob, split_sizes,
                      group_offsets, row_to_slot, slot_to_row, prob_perm, xq, xq_sf, xq_col, xq_col_sf, workspace,
                      workspace_bytes, stream=0):
    _check("moe_route_permute", _lib.moe_route_permute(
        logits, logits_dtype, x, T, H, k, E, rows_cap, topk_idx, topk_prob, split_sizes, group_offsets,
        row_to_slot, slot_to_row, prob_perm, xq, xq_sf, xq_col, xq_col_sf, workspace, workspace_bytes, stream))


def moe_grouped_mlp_bwd(w2tq, w2tsf, w1tq, w1tsf, T, H, I, E, k, rows_cap, split_sizes, group_offsets,
                        row_to_slot, slot_to_row, prob_perm, dY, saved_a, x, dX, dW1,
                        dW2, dprob, workspace, workspace_bytes, stream=0):
    _check("moe_grouped_mlp_bwd", _lib.moe_grouped_mlp_bwd(
        w2tq, w2tsf, w1tq, w1tsf, T, H, I, E, k, rows_cap, split_sizes, group_offsets, row_to_slot,
        slot_to_row, prob_perm, dY, saved_a, x, dX, dW1, dW2, dprob, workspace,
        workspace_bytes, stream))


def moe_get_device_status(stream=0) -> int:
    return _lib.moe_get_device_status(stream)


def moe_launch_count(reset: bool = False) -> int:
    return _lib.moe_launch_count(1 if reset else 0)


def moe_selftest_wait_timeout(wait_ms: int, stream=0) -> int:
    return _lib.moe_selftest_wait_timeout(wait_ms, stream)


def moe_timing_enable(on: bool) -> bool:
    return bool(_lib.moe_timing_enable(1 if on else 0))


def moe_timing_read(max_entries: int = 64) -> dict:
    """{kernel tag: (total ms, launches)} since the last read."""
    buf = ctypes.create_string_buffer(8192)
    ms = (ctypes.c_double * max_entries)()
    cnt = (_I64 * max_entries)()
    n = _lib.moe_timing_read(buf, len(buf), ms, cnt, max_entries)
    names = buf.value.decode().split("\n")[:n]
    return {names[i]: (ms[i], int(cnt[i])) for i in range(n)}
