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
