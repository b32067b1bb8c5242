"""Plain <-> blocked scale conversion on the GPU (through the C ABI): the
blocked image of plain scale bytes reads back as those bytes through the
tests' reader of the layout, its padding bytes are zero, and the library's own
scales of a quantised tensor convert back to the plain order."""
import numpy as np
import pytest

from .mxutil import sf_padding_offsets, sf_unblock

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mxfp8_grouped_gemm_x32_b200 import lib  # noqa: F401  (fails loudly if not built)
    return torch


@pytest.mark.parametrize("groups,rows,k,pad", [(1, 128, 128, 0), (3, 200, 2880, 7), (2, 5, 96, 0),
                                               (1, 1000, 4096, 16)])
def test_to_blocked_and_back(torch_cuda, groups, rows, k, pad):
    torch = torch_cuda
    from mxfp8_grouped_gemm_x32_b200 import lib
    nkb = k // 32
    ld = nkb + pad
    rng = np.random.default_rng(groups * 31 + rows)
    plain = rng.integers(0, 256, (groups * rows, ld), dtype=np.uint8)
    dplain = torch.from_numpy(plain).cuda()
    nsf = lib.moe_mx_scale_bytes(groups, rows, k)
    blocked = torch.full((nsf,), 0xAB, dtype=torch.uint8, device="cuda")
    lib.moe_mx_scales_to_blocked(dplain.data_ptr(), groups, rows, k, ld, blocked.data_ptr(), 0)
    back = torch.full((groups * rows, ld), 0xCD, dtype=torch.uint8, device="cuda")
    lib.moe_mx_scales_from_blocked(blocked.data_ptr(), groups, rows, k, back.data_ptr(), ld, 0)
    torch.cuda.synchronize()
    b = blocked.cpu().numpy()
    assert np.array_equal(sf_unblock(b, groups, rows, k).reshape(groups * rows, nkb), plain[:, :nkb])
    assert np.all(b[sf_padding_offsets(groups, rows, k)] == 0)
    bk = back.cpu().numpy()
    assert np.array_equal(bk[:, :nkb], plain[:, :nkb])
    assert np.all(bk[:, nkb:] == 0xCD)                     # bytes past k/32 of a row are left alone


def test_library_scales_read_back_plain(torch_cuda):
    torch = torch_cuda
    from mxfp8_grouped_gemm_x32_b200 import lib
    from mxfp8_grouped_gemm_x32_b200.workloads import bf16_bits_from_f32
    rows, cols = 300, 2880
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((rows, cols)) * np.exp2(rng.integers(-20, 20, (rows, 1)))).astype(np.float32)
    src = torch.from_numpy(bf16_bits_from_f32(x).view(np.int16)).view(torch.bfloat16).cuda()
    q = torch.empty(rows * cols, dtype=torch.uint8, device="cuda")
    sf = torch.empty(lib.moe_mx_scale_bytes(1, rows, cols), dtype=torch.uint8, device="cuda")
    lib.moe_mlp_quantize_mxfp8(src.data_ptr(), 1, rows, cols, lib.MOE_QUANT_ROW, q.data_ptr(), sf.data_ptr(), 0)
    plain = torch.empty(rows, cols // 32, dtype=torch.uint8, device="cuda")
    lib.moe_mx_scales_from_blocked(sf.data_ptr(), 1, rows, cols, plain.data_ptr(), cols // 32, 0)
    torch.cuda.synchronize()
    assert np.array_equal(plain.cpu().numpy(), sf_unblock(sf.cpu().numpy(), 1, rows, cols)[0])
