"""Per-tensor FP8 recipe of the layer forward (float64 + float32 numpy).
Test infrastructure only: nothing on the product path imports this.

"Efficient MoE Training for Biological Foundation Models", Challenge 2,
contrasts MXFP8 (one scaling factor per block of 32 values) with FP8 scaled
per tensor: one factor for a whole tensor.  The pages give no formula; the
readings taken here:

* element type E4M3 (the MXFP8 codec's: RNE, saturating at +-448);
* one float32 factor per tensor, computed from the tensor's current amax:
  scale = float32(448) / float32(amax), rounded as IEEE float32 division,
  clamped to the largest finite float32 (amax below ~1.3e-36); amax = 0 or
  not finite -> scale = 1;
* code = E4M3(float32(v * scale)), the product rounded to float32 first;
  value = E4M3 value / scale;
* tensors: x (all T tokens, one factor), each expert's W_gate_up [2I, H]
  and W_down [H, I] (one factor per expert matrix), and h over all routed
  rows (one factor);
* as in the BF16 recipe, h is held in bf16 between the two GEMMs (rounded
  once from its exact value), and its factor comes from that bf16 tensor;
* the combine is the plain sum of a token's k rows, out rounded to bf16.

Backward (the same recipe's training step; the pages give no formula, the
readings taken):
* the forward keeps A rounded to bf16 (as the other recipes) and its
  factors of x and of the weights; the backward reuses them (the weights
  and x have not changed in between), so W_down^T and W_gate_up^T carry the
  forward's codes, transposed (a per-tensor code does not depend on the
  layout), and wgrad1 reads x's forward codes;
* dY gets its own factor (all T tokens);
* dh = deq(dY) deq(W_down) per expert; g, u, the ScaledSwiGLU backward and
  d(prob) as in the MXFP8 recipe, from the saved A;
* da = [dg, du] and the recomputed h = p*s*u are held in bf16 (rounded once
  from their exact values), each with one factor from its bf16 tensor over
  all routed rows;
* dW_down_e = deq(dY_e)^T deq(h_e), dx = deq(da) deq(W_gate_up_e),
  dW_gate_up_e = deq(da_e)^T deq(x_e); dX sums a token's k rows.
"""
from __future__ import annotations

import numpy as np

from . import moe
from .mxfp8 import E4M3_MAX, e4m3_decode, e4m3_encode


def tensor_scale(v: np.ndarray) -> np.float32:
    """float32 factor 448 / amax of a whole tensor (1 for amax 0 or non-finite)."""
    amax = float(np.max(np.abs(np.asarray(v, dtype=np.float64)))) if np.size(v) else 0.0
    if amax == 0.0 or not np.isfinite(amax):
        return np.float32(1.0)
    with np.errstate(over="ignore"):
        s = np.float32(E4M3_MAX) / np.float32(amax)
    return s if np.isfinite(s) else np.finfo(np.float32).max


def quantize_tensor(v: np.ndarray, scale) -> np.ndarray:
    """E4M3 codes of float32(v * scale) (v holds float32-representable values)."""
    prod = np.asarray(v, dtype=np.float64).astype(np.float32) * np.float32(scale)
    return e4m3_encode(prod.astype(np.float64))


def dequantize_tensor(codes: np.ndarray, scale) -> np.ndarray:
    return e4m3_decode(codes) / np.float64(np.float32(scale))


def forward(x, w1, w2, topk_idx, topk_prob):
    """Forward of the per-tensor FP8 recipe.  Inputs as for ``moe.forward``.

    Returns a dict with the permutation, the factors (s_x, s_w1[E], s_w2[E],
    s_h), the codes of x (token order), W_gate_up, W_down and h (permuted
    rows), A, h in bf16, Y and out (float64 and bf16 bits)."""
    x = np.asarray(x, dtype=np.float64)
    w1 = np.asarray(w1, dtype=np.float64)
    w2 = np.asarray(w2, dtype=np.float64)
    T, H = x.shape
    E, I2, _ = w1.shape
    I = I2 // 2
    k = topk_idx.shape[1]
    perm, split = moe.permute(topk_idx, E)
    offs = moe.offsets(split)
    tok = perm // k
    p = np.asarray(topk_prob, dtype=np.float64).reshape(-1)[perm]
    R = perm.size

    s_x = tensor_scale(x)
    xq = quantize_tensor(x, s_x)                                  # token order
    xd = dequantize_tensor(xq, s_x)
    s_w1 = np.array([tensor_scale(w1[e]) for e in range(E)], np.float32)
    s_w2 = np.array([tensor_scale(w2[e]) for e in range(E)], np.float32)
    w1q = np.stack([quantize_tensor(w1[e], s_w1[e]) for e in range(E)])
    w2q = np.stack([quantize_tensor(w2[e], s_w2[e]) for e in range(E)])

    A = np.zeros((R, I2))
    h = np.zeros((R, I))
    for e in range(E):
        r0, r1 = offs[e], offs[e + 1]
        if r1 == r0:
            continue
        A[r0:r1] = xd[tok[r0:r1]] @ dequantize_tensor(w1q[e], s_w1[e]).T   # gate_up GEMM
        g, u = A[r0:r1, :I], A[r0:r1, I:]
        h[r0:r1] = moe.bf16_round(p[r0:r1, None] * moe.silu(g) * u)       # ScaledSwiGLU, held in bf16
    s_h = tensor_scale(h)
    hq = quantize_tensor(h, s_h)
    hd = dequantize_tensor(hq, s_h)
    Y = np.zeros((R, w2.shape[1]))
    for e in range(E):
        r0, r1 = offs[e], offs[e + 1]
        if r1 > r0:
            Y[r0:r1] = hd[r0:r1] @ dequantize_tensor(w2q[e], s_w2[e]).T  # down GEMM
    slot_row = np.empty(R, np.int64)
    slot_row[perm] = np.arange(R)
    out = Y[slot_row].reshape(T, k, -1).sum(axis=1)                     # combine
    return {"perm": perm, "split_sizes": split, "offsets": offs, "tok": tok, "p": p,
            "s_x": s_x, "s_w1": s_w1, "s_w2": s_w2, "s_h": s_h,
            "xq": xq, "w1q": w1q, "w2q": w2q, "hq": hq, "A": A, "saved": moe.bf16_round(A), "h": h, "Y": Y,
            "out": out, "out_bf16": moe.bf16_bits(out), "slot_row": slot_row}


def backward(fwd, dy, topk_prob):
    """Backward of the per-tensor FP8 recipe given ``forward``'s dict and
    dy [T, H] (bf16 values).

    Returns dX [T, H], dW1 [E, 2I, H], dW2 [E, H, I] (float64 and bf16 bits),
    dprob float32 [T, k] (slot order), the factors s_dy, s_da, s_hb and the
    intermediates dh, da (bf16), h_b (bf16) per permuted row."""
    dy = np.asarray(dy, dtype=np.float64)
    T, H = dy.shape
    E, I2, _ = fwd["w1q"].shape
    I = I2 // 2
    k = np.asarray(topk_prob).shape[1]
    perm, offs, tok, p = fwd["perm"], fwd["offsets"], fwd["tok"], fwd["p"]
    R = perm.size
    a = fwd["saved"]

    s_dy = tensor_scale(dy)
    dyd = dequantize_tensor(quantize_tensor(dy, s_dy), s_dy)                # token order
    xd = dequantize_tensor(fwd["xq"], fwd["s_x"])
    w1d = [dequantize_tensor(fwd["w1q"][e], fwd["s_w1"][e]) for e in range(E)]
    w2d = [dequantize_tensor(fwd["w2q"][e], fwd["s_w2"][e]) for e in range(E)]

    dh = np.zeros((R, I))
    da = np.zeros((R, I2))
    hb = np.zeros((R, I))
    dp_rows = np.zeros(R)
    for e in range(E):
        r0, r1 = offs[e], offs[e + 1]
        if r1 == r0:
            continue
        dh[r0:r1] = dyd[tok[r0:r1]] @ w2d[e]                              # dgrad2, contraction over H
        g, u = a[r0:r1, :I], a[r0:r1, I:]
        pe = p[r0:r1, None]
        sg = moe.sigmoid(g)
        sv = g * sg
        d = dh[r0:r1]
        da[r0:r1, :I] = moe.bf16_round(d * pe * u * sg * (1.0 + g * (1.0 - sg)))
        da[r0:r1, I:] = moe.bf16_round(d * pe * sv)
        hb[r0:r1] = moe.bf16_round(pe * sv * u)
        dp_rows[r0:r1] = np.sum(d * sv * u, axis=1)
    s_da = tensor_scale(da)
    s_hb = tensor_scale(hb)
    dad = dequantize_tensor(quantize_tensor(da, s_da), s_da)
    hbd = dequantize_tensor(quantize_tensor(hb, s_hb), s_hb)

    dW1 = np.zeros((E, I2, H))
    dW2 = np.zeros((E, H, I))
    dxr = np.zeros((R, H))
    for e in range(E):
        r0, r1 = offs[e], offs[e + 1]
        if r1 == r0:
            continue                                                       # dW_e stays 0
        dW2[e] = dyd[tok[r0:r1]].T @ hbd[r0:r1]                           # wgrad2, over the group's tokens
        dxr[r0:r1] = dad[r0:r1] @ w1d[e]                                   # dgrad1, contraction over 2I
        dW1[e] = dad[r0:r1].T @ xd[tok[r0:r1]]                            # wgrad1, over the group's tokens
    dX = np.zeros((T, H))
    np.add.at(dX, tok, dxr)
    dprob = np.zeros(T * k)
    dprob[perm] = dp_rows
    return {"dX": dX, "dX_bf16": moe.bf16_bits(dX), "dW1": dW1, "dW1_bf16": moe.bf16_bits(dW1),
            "dW2": dW2, "dW2_bf16": moe.bf16_bits(dW2),
            "dprob": dprob.reshape(T, k).astype(np.float32), "dprob_f64": dprob.reshape(T, k),
            "s_dy": s_dy, "s_da": s_da, "s_hb": s_hb, "dh": dh, "da": da, "h_b": hb, "dx_rows": dxr}
