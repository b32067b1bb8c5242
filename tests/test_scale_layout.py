"""The blocked E8M0 scale layout of the C ABI (include/moe_mxfp8.h: 512-byte
atoms of 128 rows x 4 blocks, offset ((g*RT + r/128)*KT + kb/4)*512 +
(r%32)*16 + ((r%128)/32)*4 + kb%4) is the 128x4 block-scale layout that
tcgen05 block-scaled GEMMs read.  Checked against an independent library
statement of that layout (vLLM's MXFP8 scale swizzle) through the tests'
own reader of the layout (tests/mxutil.sf_unblock), on the CPU."""
import numpy as np
import pytest

from .mxutil import sf_padding_offsets, sf_unblock


@pytest.fixture(scope="module")
def swizzle():
    try:
        from vllm.model_executor.layers.quantization.utils.mxfp8_utils import swizzle_mxfp8_scale
    except Exception as exc:  # library missing or not importable here
        pytest.skip(f"vLLM scale swizzle unavailable: {type(exc).__name__}")
    return swizzle_mxfp8_scale


@pytest.mark.parametrize("M,K", [(128, 128), (300, 640), (2880, 2880), (1, 32), (200, 4096)])
def test_blocked_layout_matches_library_swizzle(swizzle, M, K):
    import torch
    rng = np.random.default_rng(M * 7 + K)
    sf = rng.integers(0, 256, (M, K // 32), dtype=np.uint8)
    blocked = swizzle(torch.from_numpy(sf), M=M, K=K).numpy()
    RT, KT = -(-M // 128), -(-K // 128)
    assert blocked.size == RT * KT * 512
    assert np.array_equal(sf_unblock(blocked, 1, M, K)[0], sf)
    # every byte the layout does not assign to a (row, block) is padding (zero in the library's form)
    assert np.all(blocked[sf_padding_offsets(1, M, K)] == 0)
