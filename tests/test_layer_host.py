"""Host-side input checks of the Python layer (no GPU needed): the library
receives raw pointers, so tensors of the wrong type, shape or device must be
rejected before a call is made."""
import pytest
import torch

from mxfp8_grouped_gemm_x32_b200.layer import check_tensor

CPU = torch.device("cpu")


def test_accepts_a_matching_tensor():
    check_tensor(torch.zeros(4, 8, dtype=torch.int32), "idx", torch.int32, (4, 8), CPU)


@pytest.mark.parametrize("t, exc", [
    (torch.zeros(4, 8, dtype=torch.int64), TypeError),              # wrong dtype
    (torch.zeros(8, 4, dtype=torch.int32), ValueError),             # wrong shape
    (torch.zeros(4 * 8, dtype=torch.int32), ValueError),            # flattened
    (torch.zeros(8, 4, dtype=torch.int32).t(), ValueError),         # right shape, not contiguous
    (torch.zeros(4, 8, dtype=torch.int32, device="meta"), ValueError),  # another device
    ([[0] * 8] * 4, TypeError),                                     # not a tensor
])
def test_rejects(t, exc):
    with pytest.raises(exc):
        check_tensor(t, "idx", torch.int32, (4, 8), CPU)


def test_guard_allocator_detects_tail_writes():
    """The layer's guard-byte allocator (debug aid) on CPU tensors: a write
    inside a buffer leaves its guard intact, one byte past the end is named."""
    import torch
    from mxfp8_grouped_gemm_x32_b200.layer import _Alloc
    al = _Alloc(torch.device("cpu"), guard=64)
    a = al.raw(100, "a")
    b = al.typed((3, 5), torch.float32, "b")
    assert a.numel() == 112 and tuple(b.shape) == (3, 5) and b.dtype == torch.float32
    a.fill_(7)
    b.fill_(1.0)
    assert al.check() == []
    name, tail = al.tails[0]
    assert name == "a" and tail.data_ptr() == a.data_ptr() + a.numel()   # the guard starts right after a
    tail[0] = 0                                                           # a one-byte overrun of a
    assert al.check() == ["a"]
