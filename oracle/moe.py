"""Grouped MXFP8 MoE expert MLP, forward and backward, float64 numpy.
Test infrastructure only.

What the layer computes ("Efficient MoE Training for Biological Foundation
Models"):
* Challenge 1: tokens are grouped by the expert they are routed to, each
  expert gets split_sizes[e] of them, every expert's linear layers run on
  its own group, and the results are added back into token order (the
  Hugging Face loop: gather rows of an expert, run the expert, multiply by
  the routing weight, index_add into the output).
* Challenge 1 (GroupedLinear listing): gate_up has out_features =
  2 * intermediate, no bias.
* Challenge 3: Sequential(GroupedLinear(gate_up), ScaledSwiGLU(),
  GroupedLinear(down)); ScaledSwiGLU folds the routing probability
  ("scales") into the activation; every GEMM operand is quantised to
  MXFP8 before the low-precision GEMM; master weights stay in 16 bits.

Readings taken where the pages are silent:
* permutation: routed row (token t, choice j) is slot s = t*k + j; rows are
  ordered by (expert, s), i.e. a stable counting sort by expert;
* gate half first: g = A[:, :I], u = A[:, I:];
  silu(z) = z / (1 + exp(-z)); h = p * silu(g) * u;
* the routing probability is applied once, inside ScaledSwiGLU, so the
  combine is the plain sum of the k already-weighted rows of a token;
* h is quantised straight from its unrounded value (no bf16 step);
* the backward keeps A = x W1^T rounded to bf16 (the "saved activation")
  and recomputes g, u and h from it;
* backward quantisation: each GEMM operand is MXFP8 along that GEMM's K:
  dgrad2  dy along H, W2 along H;   wgrad2  dy and h along tokens;
  dgrad1  da along 2I, W1 along 2I; wgrad1  da and x along tokens;
  (blocks along tokens start at each group's first row, zero padded);
* outputs out, dX, dW1, dW2 are bf16 (round to nearest even from the
  float64 value); d(prob) is float32, in slot order [T, k].
"""
from __future__ import annotations

import numpy as np

from . import mxfp8

# ----------------------------------------------------------------------------
# bf16 conversion (the oracle's own; float64 -> bf16 with one rounding)
# ----------------------------------------------------------------------------


def bf16_round(v: np.ndarray) -> np.ndarray:
    """Round float64 to the nearest bf16 value (ties to even), returned as
    float64.  bf16: 8 significant bits, exponent range of float32,
    subnormal spacing 2^-133, overflow to infinity."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    fin = np.isfinite(a)
    a0 = np.where(fin, a, 0.0)
    _, ex = np.frexp(a0)
    e = np.maximum(ex - 1, -126)
    step = np.ldexp(1.0, e - 7)
    q = np.round(a0 / step) * step
    q = np.where(q >= 2.0 ** 128, np.inf, q)
    q = np.where(fin, q, a)
    return np.copysign(q, v)


def bf16_bits(v: np.ndarray) -> np.ndarray:
    """float64 -> bf16 bit patterns (uint16) after bf16_round."""
    q = bf16_round(v).astype(np.float32)          # exact: q is a bf16 value
    return (q.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_value(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------
# routing permutation (GroupedLinear's split_sizes)
# ----------------------------------------------------------------------------


def permute(topk_idx: np.ndarray, E: int):
    """Stable counting sort of the T*k routed slots by expert.

    Returns (perm, split_sizes): perm[r] = slot of permuted row r, rows of
    expert e are perm[offs[e]:offs[e+1]] in increasing slot order;
    split_sizes[e] = number of slots routed to e.
    """
    flat = np.asarray(topk_idx, dtype=np.int64).reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert id out of range")
    split = np.bincount(flat, minlength=E).astype(np.int64)
    perm = np.argsort(flat, kind="stable")
    return perm, split


def offsets(split) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(np.asarray(split, dtype=np.int64))])


def silu(z):
    return z / (1.0 + np.exp(-z))


def sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def _ident(v):
    return np.asarray(v, dtype=np.float64)


# ----------------------------------------------------------------------------
# forward
# ----------------------------------------------------------------------------


def forward(x, w1, w2, topk_idx, topk_prob, *, quantize=True, round_saved=True,
            experts=None, h_bf16=False):
    """Forward pass of the layer.

    x [T, H], w1 [E, 2I, H], w2 [E, H, I] as float64 values (bf16 inputs
    already converted), topk_idx int [T, k], topk_prob [T, k].
    ``quantize=False`` replaces every MXFP8 round trip by the identity;
    ``h_bf16=True`` (with ``quantize=False``: the BF16 recipe, Challenge 2's
    "BF16 uses 16 bits to represent each activation") rounds h to bf16
    between the two GEMMs;
    ``round_saved=False`` keeps the saved activation in float64.
    ``experts`` restricts the work to those experts (rows of other experts
    are left zero) -- used for sampled checks at full size.

    Returns a dict with the permutation, split_sizes, the quantised x
    (codes, scales, in permuted row order), A, the saved activation,
    quantised h, Y (per permuted row) and out (float64 and bf16 bits).
    """
    x = np.asarray(x, dtype=np.float64)
    T, H = x.shape
    E, I2, _ = w1.shape
    I = I2 // 2
    k = topk_idx.shape[1]
    perm, split = permute(topk_idx, E)
    offs = offsets(split)
    tok = perm // k
    p = np.asarray(topk_prob, dtype=np.float64).reshape(-1)[perm]
    R = perm.size
    sel = range(E) if experts is None else experts

    res = {"perm": perm, "split_sizes": split, "offsets": offs, "tok": tok, "p": p}
    xq_c = np.zeros((R, H), np.uint8)
    xq_s = np.zeros((R, H // 32), np.uint8)
    A = np.zeros((R, I2))
    hq_c = np.zeros((R, I), np.uint8)
    hq_s = np.zeros((R, I // 32), np.uint8)
    Y = np.zeros((R, w2.shape[1]))
    for e in sel:
        r0, r1 = offs[e], offs[e + 1]
        if r1 == r0:
            continue
        xg = x[tok[r0:r1]]
        if quantize:
            c, s = mxfp8.quantize_rows(xg)
            xq_c[r0:r1], xq_s[r0:r1] = c, s
            xd = mxfp8.dequantize_rows(c, s)
            w1d = mxfp8.roundtrip_rows(w1[e])
        else:
            xd, w1d = xg, _ident(w1[e])
        Ae = xd @ w1d.T                                   # gate_up GEMM
        A[r0:r1] = Ae
        g, u = Ae[:, :I], Ae[:, I:]                       # gate half first
        h = p[r0:r1, None] * silu(g) * u                  # ScaledSwiGLU
        if quantize:
            c, s = mxfp8.quantize_rows(h)                 # requantise along I
            hq_c[r0:r1], hq_s[r0:r1] = c, s
            hd = mxfp8.dequantize_rows(c, s)
            w2d = mxfp8.roundtrip_rows(w2[e])
        else:
            hd, w2d = (bf16_round(h) if h_bf16 else h), _ident(w2[e])
        Y[r0:r1] = hd @ w2d.T                             # down GEMM
    out = np.zeros((T, w2.shape[1]))
    slot_row = np.empty(R, np.int64)
    slot_row[perm] = np.arange(R)
    Ys = Y[slot_row].reshape(T, k, -1)
    for j in range(k):                                    # combine: plain sum
        out += Ys[:, j]
    res.update(xq_codes=xq_c, xq_scales=xq_s, A=A, hq_codes=hq_c, hq_scales=hq_s,
               Y=Y, out=out, out_bf16=bf16_bits(out), slot_row=slot_row)
    res["saved"] = bf16_round(A) if round_saved else A
    return res


# ----------------------------------------------------------------------------
# backward
# ----------------------------------------------------------------------------


def backward(fwd, x, w1, w2, topk_prob, dy, *, quantize=True, experts=None, bf16_held=False):
    """Backward pass given the forward's dict.

    dy [T, H] is the gradient of the combined output.  Returns dX [T, H],
    dW1 [E, 2I, H], dW2 [E, H, I] (float64 and bf16 bits) and dprob
    float32 [T, k] in slot order, plus the intermediates dh, da and h_b
    (per permuted row) for kernel-level checks.
    ``bf16_held=True`` (with ``quantize=False``: the BF16 recipe, whose
    tensors between the GEMMs are bf16) rounds da = [dg, du] and the
    recomputed h to bf16 before the GEMMs that consume them.
    """
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    T, H = x.shape
    E, I2, _ = w1.shape
    I = I2 // 2
    k = np.asarray(topk_prob).shape[1]
    perm, offs, tok, p = fwd["perm"], fwd["offsets"], fwd["tok"], fwd["p"]
    split = fwd["split_sizes"]
    R = perm.size
    a = fwd["saved"]
    sel = range(E) if experts is None else experts

    dW1 = np.zeros(w1.shape)
    dW2 = np.zeros(w2.shape)
    dxr = np.zeros((R, H))
    dh_all = np.zeros((R, I))
    da_all = np.zeros((R, I2))
    hb_all = np.zeros((R, I))
    dp_rows = np.zeros(R)
    for e in sel:
        r0, r1 = offs[e], offs[e + 1]
        if r1 == r0:
            continue                                      # dW_e stays 0
        dyg = dy[tok[r0:r1]]                              # transpose of combine
        xg = x[tok[r0:r1]]
        pe = p[r0:r1, None]
        Q = mxfp8.roundtrip_rows if quantize else _ident
        # dgrad2: dh = dy W2, contraction over H
        dh = Q(dyg) @ Q(w2[e].T).T
        # ScaledSwiGLU backward from the saved activation
        g, u = a[r0:r1, :I], a[r0:r1, I:]
        sg = sigmoid(g)
        s = g * sg
        dg = dh * pe * u * sg * (1.0 + g * (1.0 - sg))
        du = dh * pe * s
        dp_rows[r0:r1] = np.sum(dh * s * u, axis=1)
        hb = pe * s * u
        da = np.concatenate([dg, du], axis=1)
        if bf16_held:
            hb, da = bf16_round(hb), bf16_round(da)
        # wgrad2: dW2_e = dy^T h, contraction over the group's tokens
        if quantize:
            dyc = mxfp8.roundtrip_cols_grouped(dyg, [r1 - r0])[0]
            hbc = mxfp8.roundtrip_cols_grouped(hb, [r1 - r0])[0]
        else:
            dyc, hbc = dyg.T, hb.T
        dW2[e] = dyc @ hbc.T
        # dgrad1: dx = da W1, contraction over 2I
        dxr[r0:r1] = Q(da) @ Q(w1[e].T).T
        # wgrad1: dW1_e = da^T x, contraction over the group's tokens
        if quantize:
            dac = mxfp8.roundtrip_cols_grouped(da, [r1 - r0])[0]
            xc = mxfp8.roundtrip_cols_grouped(xg, [r1 - r0])[0]
        else:
            dac, xc = da.T, xg.T
        dW1[e] = dac @ xc.T
        dh_all[r0:r1], da_all[r0:r1], hb_all[r0:r1] = dh, da, hb
    dX = np.zeros((T, H))
    np.add.at(dX, tok, dxr)
    dprob = np.zeros(T * k)
    dprob[perm] = dp_rows
    return {"dX": dX, "dX_bf16": bf16_bits(dX), "dW1": dW1, "dW1_bf16": bf16_bits(dW1),
            "dW2": dW2, "dW2_bf16": bf16_bits(dW2),
            "dprob": dprob.reshape(T, k).astype(np.float32),
            "dprob_f64": dprob.reshape(T, k), "dh": dh_all, "da": da_all, "h_b": hb_all,
            "dx_rows": dxr, "split_sizes": split}
