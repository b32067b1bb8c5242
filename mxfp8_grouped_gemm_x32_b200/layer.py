"""Device buffers for one grouped MXFP8 MoE expert layer, driven through the
C ABI.  PyTorch only allocates device memory and provides the stream; every
step of the layer runs in the CUDA library (see lib.py).

Steps (names of the C entry points):
  quantize_weights  moe_mlp_quantize_weights: W_gate_up and W_down, along K
                    for the forward and along the other axis for the backward
                    (forward only: moe_mlp_quantize_mxfp8 x2)
  route             moe_router_topk: router logits -> top-k experts + probabilities
  permute           moe_permute: counting sort by expert, gather + quantise x
  forward           moe_grouped_mlp_fwd: gate_up GEMM + ScaledSwiGLU + requant,
                    down GEMM, top-k combine
  forward_bf16      moe_grouped_mlp_fwd_bf16: the same layer with bf16 operands
                    (routing from permute_index, moe_permute without x)
  backward_bf16     moe_grouped_mlp_bwd_bf16: its backward
  forward_fp8_tensor / backward_fp8_tensor
                    moe_grouped_mlp_fwd/bwd_fp8_tensor: the per-tensor FP8 recipe
  backward          moe_grouped_mlp_bwd: dgrad/wgrad of both projections,
                    ScaledSwiGLU backward, d(prob)
"""
from __future__ import annotations

import torch

from . import lib


def _ptr(t) -> int:
    return 0 if t is None else t.data_ptr()


def check_tensor(t, name: str, dtype, shape, device) -> None:
    """Raise unless `t` is a contiguous tensor of `dtype` and `shape` on
    `device`.  The library receives raw pointers, so a host tensor or a
    wrong shape must be caught here, before any kernel reads through it."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name}: expected a tensor on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


GUARD_BYTE = 0xA5


class _Alloc:
    """Device buffers of one layer.  With guard > 0 every buffer is followed
    by `guard` bytes of a fixed pattern (a debug aid: check() names every
    buffer whose tail was written, i.e. a write past its end)."""

    def __init__(self, dev, guard: int = 0):
        self.dev, self.guard = dev, (guard + 255) // 256 * 256
        self.tails = []

    def raw(self, nbytes: int, name: str) -> torch.Tensor:
        # 256-byte aligned by the caching allocator; sizes rounded to 16 bytes
        n = max(16, (nbytes + 15) // 16 * 16)
        if not self.guard:
            return torch.empty(n, dtype=torch.uint8, device=self.dev)
        n256 = (n + 255) // 256 * 256
        buf = torch.empty(n256 + self.guard, dtype=torch.uint8, device=self.dev)
        buf[n:].fill_(GUARD_BYTE)
        self.tails.append((name, buf[n:]))
        return buf[:n]

    def typed(self, shape, dtype, name: str) -> torch.Tensor:
        numel = 1
        for d in shape:
            numel *= d
        esz = torch.empty(0, dtype=dtype).element_size()
        return self.raw(numel * esz, name)[: numel * esz].view(dtype).view(*shape)

    def check(self):
        """Names of the buffers whose guard bytes changed."""
        return [name for name, t in self.tails if not bool((t == GUARD_BYTE).all())]


class GroupedMLP:
    """One layer: T tokens, hidden H, intermediate I, E experts, top-k."""

    def __init__(self, T: int, H: int, I: int, E: int, k: int, device="cuda", backward: bool = True,
                 guard: int = 0):
        self.T, self.H, self.I, self.E, self.k = T, H, I, E, k
        self.dev = torch.device(device)
        al = self._alloc = _Alloc(self.dev, guard)
        u8 = al.raw
        self.rows_cap = lib.moe_padded_rows(T, k, E)
        rc = self.rows_cap
        sb = lib.moe_mx_scale_bytes
        # quantised weights (forward: along H for gate_up, along I for down)
        self.w1q = u8(2 * E * I * H, "w1q")
        self.w1sf = u8(sb(2 * E, I, H), "w1sf")
        self.w2q = u8(E * H * I, "w2q")
        self.w2sf = u8(sb(E, H, I), "w2sf")
        # routing
        self.split_sizes = al.typed((E,), torch.int32, "split_sizes")
        self.group_offsets = al.typed((E + 1,), torch.int32, "group_offsets")
        self.row_to_slot = al.typed((rc,), torch.int32, "row_to_slot")
        self.slot_to_row = al.typed((T * k,), torch.int32, "slot_to_row")
        self.topk_idx = al.typed((T, k), torch.int32, "topk_idx")        # router outputs
        self.topk_prob = al.typed((T, k), torch.float32, "topk_prob")
        self.prob_perm = al.typed((rc,), torch.float32, "prob_perm")
        self.xq = u8(rc * H, "xq")
        self.xq_sf = u8(sb(1, rc, H), "xq_sf")
        self.hq = u8(rc * I, "hq")
        self.hq_sf = u8(sb(1, rc, I), "hq_sf")
        self.out = al.typed((T, H), torch.bfloat16, "out")
        self.dev = self.out.device      # concrete device (index resolved) for the input checks
        self.ws_perm_bytes = lib.moe_workspace_size(lib.MOE_OP_PERMUTE, T, k, E, H, I)
        self.ws_fwd_bytes = lib.moe_workspace_size(lib.MOE_OP_FWD, T, k, E, H, I)
        self.ws_perm = u8(self.ws_perm_bytes, "ws_perm")
        self.ws_fwd = u8(self.ws_fwd_bytes, "ws_fwd")
        self.backward_enabled = backward
        if backward:
            self.w1tq = u8(E * H * 2 * I, "w1tq")
            self.w1tsf = u8(sb(E, H, 2 * I), "w1tsf")
            self.w2tq = u8(E * I * H, "w2tq")
            self.w2tsf = u8(sb(E, I, H), "w2tsf")
            self.saved_a = al.typed((rc, 2 * I), torch.bfloat16, "saved_a")
            self.dX = al.typed((T, H), torch.bfloat16, "dX")
            self.dW1 = al.typed((E, 2 * I, H), torch.bfloat16, "dW1")
            self.dW2 = al.typed((E, H, I), torch.bfloat16, "dW2")
            self.dprob = al.typed((T, k), torch.float32, "dprob")
            self.ws_bwd_bytes = lib.moe_workspace_size(lib.MOE_OP_BWD, T, k, E, H, I)
            self.ws_bwd = u8(self.ws_bwd_bytes, "ws_bwd")
        else:
            self.saved_a = None
        self.xq_col = self.xq_col_sf = None   # x along tokens: only when permute(..., with_cols=True)
        self._x = None                         # the input of the last permutation (the backward's x)

    def _cols(self, with_cols: bool):
        """Buffers of the optional column form of x (x^T quantised along
        tokens in permuted order); the backward does not need them."""
        if not with_cols:
            return 0, 0
        if self.xq_col is None:
            self.xq_col = self._alloc.raw(self.H * self.rows_cap, "xq_col")
            self.xq_col_sf = self._alloc.raw(lib.moe_mx_scale_bytes(1, self.H, self.rows_cap), "xq_col_sf")
        return _ptr(self.xq_col), _ptr(self.xq_col_sf)

    def permute_index(self, topk_idx: torch.Tensor, topk_prob: torch.Tensor) -> None:
        """Routing outputs of the permutation only (no quantisation of x):
        what the BF16 forward needs."""
        check_tensor(topk_idx, "topk_idx", torch.int32, (self.T, self.k), self.dev)
        check_tensor(topk_prob, "topk_prob", torch.float32, (self.T, self.k), self.dev)
        lib.moe_permute(0, topk_idx.data_ptr(), topk_prob.data_ptr(), self.T, self.H, self.k, self.E, self.rows_cap,
                        _ptr(self.split_sizes), _ptr(self.group_offsets), _ptr(self.row_to_slot),
                        _ptr(self.slot_to_row), _ptr(self.prob_perm), 0, 0, 0, 0, _ptr(self.ws_perm),
                        self.ws_perm_bytes, self._stream())

    def forward_bf16(self, x: torch.Tensor, w1: torch.Tensor, w2: torch.Tensor) -> torch.Tensor:
        """BF16 recipe forward (moe_grouped_mlp_fwd_bf16) on the routing of
        the last permute / permute_index: x bf16 [T, H], w1 bf16 [E, 2I, H],
        w2 bf16 [E, H, I] -> out."""
        E, H, I = self.E, self.H, self.I
        check_tensor(x, "x", torch.bfloat16, (self.T, H), self.dev)
        check_tensor(w1, "w_gate_up", torch.bfloat16, (E, 2 * I, H), self.dev)
        check_tensor(w2, "w_down", torch.bfloat16, (E, H, I), self.dev)
        if getattr(self, "ws_bf16", None) is None:
            self.ws_bf16_bytes = lib.moe_workspace_size(lib.MOE_OP_FWD_BF16, self.T, self.k, E, H, I)
            self.ws_bf16 = self._alloc.raw(self.ws_bf16_bytes, "ws_bf16")
        lib.moe_grouped_mlp_fwd_bf16(w1.data_ptr(), w2.data_ptr(), self.T, H, I, E, self.k, self.rows_cap,
                                     _ptr(self.split_sizes), _ptr(self.group_offsets), _ptr(self.row_to_slot),
                                     _ptr(self.slot_to_row), _ptr(self.prob_perm), x.data_ptr(), _ptr(self.out),
                                     _ptr(self.saved_a), _ptr(self.ws_bf16), self.ws_bf16_bytes, self._stream())
        return self.out

    def backward_bf16(self, dY: torch.Tensor, x: torch.Tensor, w1: torch.Tensor, w2: torch.Tensor):
        """BF16 recipe backward (moe_grouped_mlp_bwd_bf16) after forward_bf16
        on the same routing: dY, x bf16 [T, H], w1 bf16 [E, 2I, H], w2 bf16
        [E, H, I] -> (dX, dW1, dW2, dprob)."""
        if not self.backward_enabled:
            raise RuntimeError("this layer was built with backward=False")
        E, H, I = self.E, self.H, self.I
        check_tensor(dY, "dY", torch.bfloat16, (self.T, H), self.dev)
        check_tensor(x, "x", torch.bfloat16, (self.T, H), self.dev)
        check_tensor(w1, "w_gate_up", torch.bfloat16, (E, 2 * I, H), self.dev)
        check_tensor(w2, "w_down", torch.bfloat16, (E, H, I), self.dev)
        if getattr(self, "ws_bwd_bf16", None) is None:
            self.ws_bwd_bf16_bytes = lib.moe_workspace_size(lib.MOE_OP_BWD_BF16, self.T, self.k, E, H, I)
            self.ws_bwd_bf16 = self._alloc.raw(self.ws_bwd_bf16_bytes, "ws_bwd_bf16")
        lib.moe_grouped_mlp_bwd_bf16(w1.data_ptr(), w2.data_ptr(), self.T, H, I, E, self.k, self.rows_cap,
                                     _ptr(self.split_sizes), _ptr(self.group_offsets), _ptr(self.row_to_slot),
                                     _ptr(self.slot_to_row), _ptr(self.prob_perm), dY.data_ptr(),
                                     _ptr(self.saved_a), x.data_ptr(), _ptr(self.dX), _ptr(self.dW1),
                                     _ptr(self.dW2), _ptr(self.dprob), _ptr(self.ws_bwd_bf16),
                                     self.ws_bwd_bf16_bytes, self._stream())
        return self.dX, self.dW1, self.dW2, self.dprob

    def forward_fp8_tensor(self, x: torch.Tensor, w1: torch.Tensor, w2: torch.Tensor) -> torch.Tensor:
        """Per-tensor FP8 recipe forward (moe_grouped_mlp_fwd_fp8_tensor) on
        the routing of the last permute / permute_index: x bf16 [T, H], w1
        bf16 [E, 2I, H], w2 bf16 [E, H, I] -> out; the factors land in
        self.fp8_scales (x, h, W_gate_up[E], W_down[E])."""
        E, H, I = self.E, self.H, self.I
        check_tensor(x, "x", torch.bfloat16, (self.T, H), self.dev)
        check_tensor(w1, "w_gate_up", torch.bfloat16, (E, 2 * I, H), self.dev)
        check_tensor(w2, "w_down", torch.bfloat16, (E, H, I), self.dev)
        if getattr(self, "ws_f8t", None) is None:
            self.ws_f8t_bytes = lib.moe_workspace_size(lib.MOE_OP_FWD_FP8_TENSOR, self.T, self.k, E, H, I)
            self.ws_f8t = self._alloc.raw(self.ws_f8t_bytes, "ws_f8t")
            self.fp8_scales = self._alloc.typed((2 + 2 * E,), torch.float32, "fp8_scales")
        lib.moe_grouped_mlp_fwd_fp8_tensor(w1.data_ptr(), w2.data_ptr(), self.T, H, I, E, self.k, self.rows_cap,
                                           _ptr(self.split_sizes), _ptr(self.group_offsets), _ptr(self.row_to_slot),
                                           _ptr(self.slot_to_row), _ptr(self.prob_perm), x.data_ptr(),
                                           _ptr(self.out), _ptr(self.saved_a), _ptr(self.fp8_scales),
                                           _ptr(self.ws_f8t), self.ws_f8t_bytes, self._stream())
        return self.out

    def backward_fp8_tensor(self, dY: torch.Tensor, x: torch.Tensor, w1: torch.Tensor, w2: torch.Tensor):
        """Per-tensor FP8 recipe backward (moe_grouped_mlp_bwd_fp8_tensor)
        after forward_fp8_tensor on the same routing, x and weights -> (dX,
        dW1, dW2, dprob); the factors of dY, da and h land in
        self.fp8_bwd_scales."""
        if not self.backward_enabled:
            raise RuntimeError("this layer was built with backward=False")
        if getattr(self, "fp8_scales", None) is None:
            raise RuntimeError("backward_fp8_tensor needs forward_fp8_tensor first")
        E, H, I = self.E, self.H, self.I
        check_tensor(dY, "dY", torch.bfloat16, (self.T, H), self.dev)
        check_tensor(x, "x", torch.bfloat16, (self.T, H), self.dev)
        check_tensor(w1, "w_gate_up", torch.bfloat16, (E, 2 * I, H), self.dev)
        check_tensor(w2, "w_down", torch.bfloat16, (E, H, I), self.dev)
        if getattr(self, "ws_bwd_f8t", None) is None:
            self.ws_bwd_f8t_bytes = lib.moe_workspace_size(lib.MOE_OP_BWD_FP8_TENSOR, self.T, self.k, E, H, I)
            self.ws_bwd_f8t = self._alloc.raw(self.ws_bwd_f8t_bytes, "ws_bwd_f8t")
            self.fp8_bwd_scales = self._alloc.typed((3,), torch.float32, "fp8_bwd_scales")
        lib.moe_grouped_mlp_bwd_fp8_tensor(w1.data_ptr(), w2.data_ptr(), self.T, H, I, E, self.k, self.rows_cap,
                                           _ptr(self.split_sizes), _ptr(self.group_offsets), _ptr(self.row_to_slot),
                                           _ptr(self.slot_to_row), _ptr(self.prob_perm), dY.data_ptr(),
                                           _ptr(self.saved_a), x.data_ptr(), _ptr(self.fp8_scales), _ptr(self.dX),
                                           _ptr(self.dW1), _ptr(self.dW2), _ptr(self.dprob),
                                           _ptr(self.fp8_bwd_scales), _ptr(self.ws_bwd_f8t), self.ws_bwd_f8t_bytes,
                                           self._stream())
        return self.dX, self.dW1, self.dW2, self.dprob

    def check_guards(self):
        """Names of the buffers written past their end (layers built with
        guard > 0; always empty otherwise)."""
        return self._alloc.check()

    @staticmethod
    def _stream() -> int:
        return torch.cuda.current_stream().cuda_stream

    def quantize_weights(self, w1: torch.Tensor, w2: torch.Tensor) -> None:
        """w1 bf16 [E, 2I, H] (gate rows first), w2 bf16 [E, H, I]."""
        E, H, I, s = self.E, self.H, self.I, self._stream()
        check_tensor(w1, "w_gate_up", torch.bfloat16, (E, 2 * I, H), self.dev)
        check_tensor(w2, "w_down", torch.bfloat16, (E, H, I), self.dev)
        if self.backward_enabled:
            # both directions of both weights from one read of each
            lib.moe_mlp_quantize_weights(w1.data_ptr(), w2.data_ptr(), E, H, I, _ptr(self.w1q), _ptr(self.w1sf),
                                         _ptr(self.w2q), _ptr(self.w2sf), _ptr(self.w1tq), _ptr(self.w1tsf),
                                         _ptr(self.w2tq), _ptr(self.w2tsf), s)
            return
        lib.moe_mlp_quantize_mxfp8(w1.data_ptr(), 2 * E, I, H, lib.MOE_QUANT_ROW, _ptr(self.w1q), _ptr(self.w1sf), s)
        lib.moe_mlp_quantize_mxfp8(w2.data_ptr(), E, H, I, lib.MOE_QUANT_ROW, _ptr(self.w2q), _ptr(self.w2sf), s)

    def route(self, logits: torch.Tensor):
        """Router logits fp32 or bf16 [T, E] -> (topk_idx int32 [T, k],
        topk_prob float32 [T, k]) in this layer's routing buffers."""
        dt = {torch.float32: lib.MOE_DTYPE_F32, torch.bfloat16: lib.MOE_DTYPE_BF16}.get(logits.dtype)
        if dt is None:
            raise TypeError(f"logits: expected float32 or bfloat16, got {logits.dtype}")
        check_tensor(logits, "logits", logits.dtype, (self.T, self.E), self.dev)
        lib.moe_router_topk(logits.data_ptr(), dt, self.T, self.E, self.k, _ptr(self.topk_idx),
                            _ptr(self.topk_prob), self._stream())
        return self.topk_idx, self.topk_prob

    def route_permute(self, logits: torch.Tensor, x: torch.Tensor, with_cols: bool = False):
        """Router and permutation in one call (moe_route_permute): logits fp32
        or bf16 [T, E], x bf16 [T, H]; the routing lands in topk_idx /
        topk_prob, the quantised x in this layer's buffers."""
        dt = {torch.float32: lib.MOE_DTYPE_F32, torch.bfloat16: lib.MOE_DTYPE_BF16}.get(logits.dtype)
        if dt is None:
            raise TypeError(f"logits: expected float32 or bfloat16, got {logits.dtype}")
        check_tensor(logits, "logits", logits.dtype, (self.T, self.E), self.dev)
        check_tensor(x, "x", torch.bfloat16, (self.T, self.H), self.dev)
        xc, xcs = self._cols(with_cols)
        lib.moe_route_permute(logits.data_ptr(), dt, x.data_ptr(), self.T, self.H, self.k, self.E, self.rows_cap,
                              _ptr(self.topk_idx), _ptr(self.topk_prob), _ptr(self.split_sizes),
                              _ptr(self.group_offsets), _ptr(self.row_to_slot), _ptr(self.slot_to_row),
                              _ptr(self.prob_perm), _ptr(self.xq), _ptr(self.xq_sf), xc, xcs, _ptr(self.ws_perm),
                              self.ws_perm_bytes, self._stream())
        self._x = x
        return self.topk_idx, self.topk_prob

    def permute(self, x: torch.Tensor, topk_idx: torch.Tensor, topk_prob: torch.Tensor,
                with_cols: bool = False) -> None:
        """x bf16 [T, H]; topk_idx int32 [T, k]; topk_prob float32 [T, k].
        with_cols also writes x^T quantised along tokens (xq_col), which the
        backward makes for itself from x."""
        check_tensor(x, "x", torch.bfloat16, (self.T, self.H), self.dev)
        check_tensor(topk_idx, "topk_idx", torch.int32, (self.T, self.k), self.dev)
        check_tensor(topk_prob, "topk_prob", torch.float32, (self.T, self.k), self.dev)
        xc, xcs = self._cols(with_cols)
        lib.moe_permute(x.data_ptr(), topk_idx.data_ptr(), topk_prob.data_ptr(), self.T, self.H, self.k,
                        self.E, self.rows_cap, _ptr(self.split_sizes), _ptr(self.group_offsets),
                        _ptr(self.row_to_slot), _ptr(self.slot_to_row), _ptr(self.prob_perm),
                        _ptr(self.xq), _ptr(self.xq_sf), xc, xcs, _ptr(self.ws_perm), self.ws_perm_bytes,
                        self._stream())
        self._x = x

    def forward(self) -> torch.Tensor:
        lib.moe_grouped_mlp_fwd(_ptr(self.w1q), _ptr(self.w1sf), _ptr(self.w2q), _ptr(self.w2sf), self.T,
                                self.H, self.I, self.E, self.k, self.rows_cap, _ptr(self.split_sizes),
                                _ptr(self.group_offsets), _ptr(self.row_to_slot), _ptr(self.slot_to_row),
                                _ptr(self.prob_perm), _ptr(self.xq), _ptr(self.xq_sf), _ptr(self.out),
                                _ptr(self.saved_a),
                                _ptr(self.hq), _ptr(self.hq_sf), _ptr(self.ws_fwd), self.ws_fwd_bytes,
                                self._stream())
        return self.out

    def backward(self, dY: torch.Tensor, x: torch.Tensor = None):
        """dY bf16 [T, H]; x defaults to the input of the last permutation."""
        if not self.backward_enabled:
            raise RuntimeError("this layer was built with backward=False")
        x = self._x if x is None else x
        if x is None:
            raise RuntimeError("backward needs x: call permute first or pass x")
        check_tensor(dY, "dY", torch.bfloat16, (self.T, self.H), self.dev)
        check_tensor(x, "x", torch.bfloat16, (self.T, self.H), self.dev)
        lib.moe_grouped_mlp_bwd(_ptr(self.w2tq), _ptr(self.w2tsf), _ptr(self.w1tq), _ptr(self.w1tsf),
                                self.T, self.H, self.I, self.E, self.k, self.rows_cap,
                                _ptr(self.split_sizes), _ptr(self.group_offsets), _ptr(self.row_to_slot),
                                _ptr(self.slot_to_row), _ptr(self.prob_perm), dY.data_ptr(),
                                _ptr(self.saved_a), x.data_ptr(),
                                _ptr(self.dX), _ptr(self.dW1), _ptr(self.dW2), _ptr(self.dprob),
                                _ptr(self.ws_bwd), self.ws_bwd_bytes, self._stream())
        return self.dX, self.dW1, self.dW2, self.dprob

    def step(self, x, topk_idx, topk_prob, w1, w2, dY=None):
        """One pass of the whole layer: weight quantisation, permutation,
        forward and (if dY is given) backward."""
        self.quantize_weights(w1, w2)
        self.permute(x, topk_idx, topk_prob)
        out = self.forward()
        if dY is None:
            return out
        return (out,) + tuple(self.backward(dY, x))

    def device_status(self) -> int:
        return lib.moe_get_device_status(self._stream())
