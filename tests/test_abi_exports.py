"""The C-ABI library builds for sm_100a, loads, and exports every function
declared in include/moe_mxfp8.h (no GPU needed: no compute call is made);
host-side argument checks return their error codes without a device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_mxfp8.h")


def _declared():
    with open(HEADER) as fh:
        text = fh.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def libso():
    from mxfp8_grouped_gemm_x32_b200 import build_lib
    path = build_lib.build()
    return ctypes.CDLL(path)


def test_every_declared_symbol_is_exported(libso):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(libso, n), n


def test_binding_covers_header():
    from mxfp8_grouped_gemm_x32_b200 import lib
    assert sorted(lib.EXPORTED) == _declared()


def test_host_side_sizes():
    from mxfp8_grouped_gemm_x32_b200 import lib
    assert lib.moe_padded_rows(512, 2, 4) == 1536
    assert lib.moe_padded_rows(8192, 2, 8) == 17408
    assert lib.moe_mx_scale_bytes(1, 128, 128) == 512
    assert lib.moe_mx_scale_bytes(2, 2880, 2880) == 2 * 23 * 23 * 512
    assert lib.moe_mx_scale_bytes(1, 128, 100) == -1
    assert lib.moe_workspace_size(lib.MOE_OP_FWD, 512, 2, 4, 256, 512) > 0
    assert lib.moe_workspace_size(99, 512, 2, 4, 256, 512) == -1


def test_host_side_argument_errors():
    from mxfp8_grouped_gemm_x32_b200 import lib
    # null pointers and bad modes are rejected before any device work
    assert lib._lib.moe_mlp_quantize_mxfp8(None, 1, 32, 32, 1, None, None, None) == 1
    assert lib._lib.moe_combine(None, 1, 1, 8, None, None) == 1
    assert lib.status_string(6).startswith("device: bounded")


def test_router_argument_errors():
    from mxfp8_grouped_gemm_x32_b200 import lib
    f = lib._lib.moe_router_topk
    p = 16  # a non-null dummy pointer: every case below is rejected before it is used
    assert f(None, 0, 4, 8, 2, p, p, None) == 1            # null logits
    assert f(p, 2, 4, 8, 2, p, p, None) == 1               # unknown dtype
    assert f(p, 0, 4, 8, 9, p, p, None) == 1               # k > E
    assert f(p, 0, 4, 8, 0, p, p, None) == 1               # k = 0
    assert f(p, 0, 4, 300, 2, p, p, None) == 2             # E > 256
    assert f(p, 0, 4, 64, 33, p, p, None) == 2             # k > 32


# Every case below is rejected by the host-side checks before the library
# looks for a device, so it returns the same code with or without a GPU and no
# pointer is ever dereferenced.  P is an aligned non-null dummy, M a
# misaligned one.
P, M = 1 << 20, (1 << 20) + 8
INVALID, UNSUPPORTED, WORKSPACE, TOO_LARGE = 1, 2, 3, 8


def _permute_args(T=64, H=256, k=2, E=4, rows_cap=None, x=P, xq=P, xq_col=P, xq_col_sf=P, ws=P,
                  ws_bytes=1 << 30):
    from mxfp8_grouped_gemm_x32_b200 import lib
    if rows_cap is None:
        rows_cap = lib.moe_padded_rows(T, k, E)
    return (x, P, P, T, H, k, E, rows_cap, P, P, P, P, P, xq, P, xq_col, xq_col_sf, ws, ws_bytes, None)


def test_permute_argument_errors():
    from mxfp8_grouped_gemm_x32_b200 import lib
    f = lib._lib.moe_permute
    assert f(*_permute_args(x=None)) == INVALID                      # null x with T > 0
    assert f(*_permute_args(xq_col_sf=None)) == INVALID              # column form half given
    assert f(*_permute_args(k=5, E=4)) == INVALID                    # k > E
    assert f(*_permute_args(E=300)) == UNSUPPORTED                   # E > MOE_MAX_EXPERTS
    assert f(*_permute_args(H=48)) == UNSUPPORTED                    # H % 32 != 0
    assert f(*_permute_args(T=1 << 29, k=2, rows_cap=1 << 31)) == UNSUPPORTED   # T*k >= 2^30
    assert f(*_permute_args(rows_cap=128)) == INVALID                # below moe_padded_rows
    assert f(*_permute_args(rows_cap=lib.moe_padded_rows(64, 2, 4) + 64)) == INVALID  # not a multiple of 128
    assert f(*_permute_args(xq=M)) == INVALID                        # misaligned output
    assert f(*_permute_args(ws=None)) == WORKSPACE
    assert f(*_permute_args(ws_bytes=16)) == WORKSPACE
    g = lib._lib.moe_permute_noalloc
    assert g(*_permute_args(x=None)[:17], None) == INVALID
    assert g(*_permute_args(T=1 << 29, k=2, rows_cap=1 << 31)[:17], None) == UNSUPPORTED
    T, k, E = 131073, 2, 256                                           # 257 histogram blocks x 256 experts
    assert g(*_permute_args(T=T, k=k, E=E)[:17], None) == TOO_LARGE


def _fwd_args(T=64, H=256, I=512, E=4, k=2, rows_cap=None, w1q=P, out=P, hq=P, hq_sf=P, ws=P, ws_bytes=1 << 40):
    from mxfp8_grouped_gemm_x32_b200 import lib
    if rows_cap is None:
        rows_cap = lib.moe_padded_rows(T, k, E)
    return (w1q, P, P, P, T, H, I, E, k, rows_cap, P, P, P, P, P, P, P, out, P, hq, hq_sf, ws, ws_bytes, None)


def test_forward_argument_errors():
    from mxfp8_grouped_gemm_x32_b200 import lib
    f = lib._lib.moe_grouped_mlp_fwd
    assert f(*_fwd_args(w1q=None)) == INVALID
    assert f(*_fwd_args(hq_sf=None)) == INVALID                      # hq given without its scales
    assert f(*_fwd_args(I=96)) == UNSUPPORTED                        # I % 64 != 0
    assert f(*_fwd_args(H=48)) == UNSUPPORTED
    assert f(*_fwd_args(k=5, E=4)) == UNSUPPORTED
    assert f(*_fwd_args(T=1 << 29, k=2, rows_cap=1 << 31)) == UNSUPPORTED
    assert f(*_fwd_args(rows_cap=128)) == INVALID
    assert f(*_fwd_args(out=M)) == INVALID
    assert f(*_fwd_args(ws_bytes=16)) == WORKSPACE
    need = lib.moe_workspace_size(lib.MOE_OP_FWD, 64, 2, 4, 256, 512)
    assert f(*_fwd_args(hq=None, hq_sf=None, ws_bytes=need - 1)) == WORKSPACE   # h in the workspace


def _bwd_args(T=64, H=256, I=512, E=4, k=2, saved=P, dW1=P, ws=P, ws_bytes=1 << 40):
    from mxfp8_grouped_gemm_x32_b200 import lib
    rows_cap = lib.moe_padded_rows(T, k, E)
    return (P, P, P, P, T, H, I, E, k, rows_cap, P, P, P, P, P, P, saved, P, P, dW1, P, P, ws, ws_bytes, None)


def test_backward_argument_errors():
    from mxfp8_grouped_gemm_x32_b200 import lib
    f = lib._lib.moe_grouped_mlp_bwd
    assert f(*_bwd_args(saved=None)) == INVALID
    assert f(*_bwd_args(H=48)) == UNSUPPORTED
    assert f(*_bwd_args(E=300, k=2)) == UNSUPPORTED
    assert f(*_bwd_args(dW1=M)) == INVALID
    assert f(*_bwd_args(saved=P + 16)) == INVALID                   # saved_a needs 32-byte alignment
    assert f(*_bwd_args(ws=P + 128)) == INVALID                     # workspace needs 256-byte alignment
    need = lib.moe_workspace_size(lib.MOE_OP_BWD, 64, 2, 4, 256, 512)
    assert f(*_bwd_args(ws_bytes=need - 1)) == WORKSPACE


def test_fp8_tensor_forward_argument_errors():
    from mxfp8_grouped_gemm_x32_b200 import lib
    f = lib._lib.moe_grouped_mlp_fwd_fp8_tensor
    rc = lib.moe_padded_rows(64, 2, 4)
    args = lambda H=256, ws=P, wsb=1 << 40, x=P, sc=None, sa=None: (P, P, 64, H, 512, 4, 2, rc, P, P, P, P, P, x, P,
                                                                    sa, sc, ws, wsb, None)
    assert f(*args(x=None)) == INVALID                                      # x missing with T > 0
    assert f(*args(x=M)) == INVALID                                         # misaligned x
    assert f(*args(sc=P + 2)) == INVALID                                    # misaligned factor output
    assert f(*args(sa=M)) == INVALID                                        # misaligned saved A
    assert f(*args(H=48)) == UNSUPPORTED
    need = lib.moe_workspace_size(lib.MOE_OP_FWD_FP8_TENSOR, 64, 2, 4, 256, 512)
    assert need > 0
    assert f(*args(wsb=need - 1)) == WORKSPACE
    assert f(*args(ws=P + 128)) == WORKSPACE                                # 256-byte aligned workspace


def test_quantise_and_combine_argument_errors():
    from mxfp8_grouped_gemm_x32_b200 import lib
    q = lib._lib.moe_mlp_quantize_mxfp8
    assert q(P, 1, 64, 48, lib.MOE_QUANT_ROW, P, P, None) == UNSUPPORTED    # cols % 32
    assert q(P, 1, 48, 64, lib.MOE_QUANT_COL, P, P, None) == UNSUPPORTED    # rows % 32
    assert q(P, 1, 64, 12, lib.MOE_QUANT_COL, P, P, None) == UNSUPPORTED    # cols % 8
    assert q(P, 1, 64, 64, 3, P, P, None) == INVALID                        # unknown mode
    assert q(M, 1, 64, 64, lib.MOE_QUANT_ROW, P, P, None) == INVALID
    w = lib._lib.moe_mlp_quantize_weights
    assert w(P, P, 4, 256, 512, *([P] * 7), None, None) == INVALID          # a null output
    assert w(P, M, 4, 256, 512, *([P] * 8), None) == INVALID                # misaligned input
    assert w(P, P, 0, 256, 512, *([P] * 8), None) == INVALID                # E = 0
    assert w(P, P, 4, 256, 96, *([P] * 8), None) == UNSUPPORTED             # I % 64
    c = lib._lib.moe_combine
    assert c(P, 4, 2, 12, P, None) == INVALID                                # H % 8
    assert c(P, 4, 2, 64, M, None) == INVALID
    assert c(P, -1, 2, 64, P, None) == INVALID


def test_scale_conversion_argument_errors():
    from mxfp8_grouped_gemm_x32_b200 import lib
    t = lib._lib.moe_mx_scales_to_blocked
    f = lib._lib.moe_mx_scales_from_blocked
    assert t(P, 1, 64, 48, 2, P, None) == INVALID           # k % 32
    assert t(P, 1, 64, 128, 3, P, None) == INVALID          # ld < k/32
    assert t(None, 1, 64, 128, 4, P, None) == INVALID       # null plain
    assert t(P, 1, 64, 128, 4, P + 2, None) == INVALID      # blocked not 4-byte aligned
    assert t(P, -1, 64, 128, 4, P, None) == INVALID
    assert t(None, 0, 64, 128, 4, None, None) == 0          # nothing to convert
    assert f(P, 1, 64, 48, P, 2, None) == INVALID
    assert f(P, 1, 64, 128, P, 3, None) == INVALID
    assert f(None, 1, 64, 128, P, 4, None) == INVALID
    assert f(P, 1, 0, 128, None, 4, None) == 0


def test_route_permute_argument_errors():
    from mxfp8_grouped_gemm_x32_b200 import lib
    f = lib._lib.moe_route_permute

    def args(T=64, H=256, k=2, E=4, dtype=0, logits=P, x=P, ws_bytes=1 << 30):
        rows_cap = lib.moe_padded_rows(T, k, E) if T < (1 << 28) else 1 << 31
        return (logits, dtype, x, T, H, k, E, rows_cap, P, P, P, P, P, P, P, P, P, P, P, P, ws_bytes, None)
    assert f(*args(logits=None)) == INVALID
    assert f(*args(dtype=5)) == INVALID
    assert f(*args(k=5, E=4)) == INVALID
    assert f(*args(k=33, E=64)) == UNSUPPORTED                    # router keeps at most 32
    assert f(*args(H=48)) == UNSUPPORTED
    assert f(*args(x=M)) == INVALID
    assert f(*args(ws_bytes=16)) == WORKSPACE


def _recipe_bwd_args(fp8, T=64, H=256, I=512, E=4, k=2, saved=P, x=P, dW1=P, fs=P, sc=None, ws=P, ws_bytes=1 << 40):
    from mxfp8_grouped_gemm_x32_b200 import lib
    rc = lib.moe_padded_rows(T, k, E)
    head = (P, P, T, H, I, E, k, rc, P, P, P, P, P, P, saved, x)
    tail = (P, dW1, P, P)
    if fp8:
        return head + (fs,) + tail + (sc, ws, ws_bytes, None)
    return head + tail + (ws, ws_bytes, None)


@pytest.mark.parametrize("fp8", [False, True])
def test_recipe_backward_argument_errors(fp8):
    """moe_grouped_mlp_bwd_bf16 / moe_grouped_mlp_bwd_fp8_tensor reject bad
    arguments with their documented codes before looking for a device."""
    from mxfp8_grouped_gemm_x32_b200 import lib
    f = lib._lib.moe_grouped_mlp_bwd_fp8_tensor if fp8 else lib._lib.moe_grouped_mlp_bwd_bf16
    a = lambda **kw: _recipe_bwd_args(fp8, **kw)
    assert f(*a(saved=None)) == INVALID                                     # no saved A
    assert f(*a(x=None)) == INVALID
    assert f(*a(H=48)) == UNSUPPORTED
    assert f(*a(I=96)) == UNSUPPORTED
    assert f(*a(E=300, k=2)) == UNSUPPORTED
    assert f(*a(dW1=M)) == INVALID                                          # misaligned output
    assert f(*a(saved=P + 16)) == INVALID                                   # saved A needs 32-byte alignment
    assert f(*a(ws=P + 128)) == INVALID                                     # workspace needs 256-byte alignment
    op = lib.MOE_OP_BWD_FP8_TENSOR if fp8 else lib.MOE_OP_BWD_BF16
    need = lib.moe_workspace_size(op, 64, 2, 4, 256, 512)
    assert need > 0
    assert f(*a(ws_bytes=need - 1)) == WORKSPACE
    if fp8:
        assert f(*a(fs=None)) == INVALID                                    # the forward's factors are needed
        assert f(*a(fs=P + 2)) == INVALID
        assert f(*a(sc=P + 2)) == INVALID
