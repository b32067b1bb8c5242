"""Bounds for comparing the CUDA path with the oracle where more than one
result is correct.

The kernels compute every value that gets requantised to MXFP8 (h in the
forward; da = [dg | du] and h in the backward) in fp32 from fp32 tensor-core
accumulations, the oracle in float64.  The two agree to a few fp32 ulps of
the accumulation, so an E4M3 code (or a block scale) whose oracle value lies
within that distance of a rounding boundary can legitimately come out either
way; the same holds for the bf16 rounding of the saved activation.  These
helpers compute, from ORACLE data only, for each requantised element the
largest change of its dequantised value over the codes any value inside the
error band would get (0 for unambiguous elements), and propagate it through
the following GEMM as an element-wise allowance.  No value of the CUDA path
enters a bound.

Error band of a value v produced by the kernels:
  accumulation   2^-22 * sqrt(K * sum_k t_k^2)    (t_k the K products)
  activation     2^-19 * |v|                      (fast exp / divide)
"""
from __future__ import annotations

import numpy as np

from oracle import moe as omoe
from oracle import mxfp8 as omx

ACC = 2.0 ** -22
ACT = 2.0 ** -19


def wbound(w: np.ndarray) -> np.ndarray:
    """Element-wise upper bound on |dequantised MXFP8 weight| without
    quantising: normal codes are within half a step (2^-4 relative) of |w|;
    subnormal codes within 2^-10 * 2^s, and 2^s < block amax / 224, so
    within 2^-17 of the block maximum -- bounded here by 2^-12 of the row
    maximum."""
    a = np.abs(np.asarray(w, np.float64))
    return a * (1.0 + 2.0 ** -4) + 2.0 ** -12 * a.max(axis=-1, keepdims=True)


def acc_band(a_deq: np.ndarray, b_deq: np.ndarray) -> np.ndarray:
    """Accumulation error band of a_deq @ b_deq.T (a [M,K], b [N,K])."""
    K = a_deq.shape[1]
    return ACC * np.sqrt(K * ((a_deq ** 2) @ (b_deq ** 2).T))


def code_ambiguity(v: np.ndarray, band: np.ndarray) -> np.ndarray:
    """v [M, K] quantised along K in 32-blocks; band >= 0 bounds |gpu - v|.
    Returns D [M, K]: max |deq(code of any value in [v-band, v+band]) - deq(code of v)|,
    over every scale any block amax in its band could select."""
    v = np.asarray(v, np.float64)
    M, K = v.shape
    c, s = omx.quantize_rows(v)
    ref = omx.dequantize_rows(c, s)
    vb = v.reshape(M, K // 32, 32)
    bb = np.asarray(band, np.float64).reshape(M, K // 32, 32)
    amax = np.abs(vb).max(axis=2)
    bmax = bb.max(axis=2)
    D = np.zeros((M, K // 32, 32))
    for am in (np.maximum(amax - bmax, 0.0), amax + bmax, amax):
        sb = omx.scale_exponent(am).astype(np.int64)
        inv = np.ldexp(1.0, 127 - sb)[:, :, None]
        sc = np.ldexp(1.0, sb - 127)[:, :, None]
        for w in (vb - bb, vb + bb):
            d = omx.e4m3_decode(omx.e4m3_encode(w * inv)) * sc
            D = np.maximum(D, np.abs(d - ref.reshape(M, K // 32, 32)))
    return D.reshape(M, K)


def code_ambiguity_cols(v: np.ndarray, band: np.ndarray, groups) -> list:
    """Column-wise (along tokens, 32-row blocks from each group's first row)
    version: per group, D of the transposed group [N, M_g]."""
    out, r0 = [], 0
    for m in groups:
        m = int(m)
        if m == 0:
            out.append(np.zeros((v.shape[1], 0)))
            continue
        mp = -(-m // 32) * 32
        vt = np.zeros((v.shape[1], mp))
        bt = np.zeros((v.shape[1], mp))
        vt[:, :m] = v[r0:r0 + m].T
        bt[:, :m] = band[r0:r0 + m].T
        out.append(code_ambiguity(vt, bt)[:, :m])
        r0 += m
    return out


def bf16_alternatives(a: np.ndarray, band: np.ndarray):
    """Range of bf16 values the kernel may store for a float64 value a known
    to within band: (lowest, highest); both equal bf16(a) when unambiguous."""
    return omoe.bf16_round(a - band), omoe.bf16_round(a + band)


def _rows_by_expert(offs, E):
    return [slice(offs[e], offs[e + 1]) for e in range(E)]


def forward_allowance(f, x, w1, w2, topk_idx):
    """Element-wise allowance for out [T, H] from ambiguous h codes."""
    E, I2, H = w1.shape
    I = I2 // 2
    T, k = topk_idx.shape
    allow_rows = np.zeros((f["perm"].size, w2.shape[1]))
    for e, sl in enumerate(_rows_by_expert(f["offsets"], E)):
        if sl.stop == sl.start:
            continue
        xd = omx.roundtrip_rows(x[f["tok"][sl]])
        bA = acc_band(xd, wbound(w1[e]))
        A = f["A"][sl]
        g, u = A[:, :I], A[:, I:]
        p = f["p"][sl][:, None]
        sg = omoe.sigmoid(g)
        h = p * g * sg * u
        bh = np.abs(p * u * sg * (1 + g * (1 - sg))) * bA[:, :I] + np.abs(p * g * sg) * bA[:, I:] + ACT * np.abs(h)
        Dh = code_ambiguity(h, bh)
        allow_rows[sl] = Dh @ wbound(w2[e]).T
    return allow_rows[f["slot_row"]].reshape(T, k, -1).sum(axis=1)


def backward_allowance(f, b, x, w1, w2, dy, topk_idx):
    """Element-wise allowances for dX, dW1, dW2 and dprob."""
    E, I2, H = w1.shape
    I = I2 // 2
    T, k = topk_idx.shape
    R = f["perm"].size
    allow_dx = np.zeros((R, H))
    allow_dp = np.zeros(R)
    aW1 = np.zeros(w1.shape)
    aW2 = np.zeros(w2.shape)
    for e, sl in enumerate(_rows_by_expert(f["offsets"], E)):
        m = sl.stop - sl.start
        if m == 0:
            continue
        tok = f["tok"][sl]
        p = f["p"][sl][:, None]
        # saved activation: bf16 of A, A known to within its accumulation band
        xd = omx.roundtrip_rows(x[tok])
        bA = acc_band(xd, wbound(w1[e]))
        lo, hi = bf16_alternatives(f["A"][sl], bA)
        a = f["saved"][sl]
        g, u = a[:, :I], a[:, I:]
        # dh = dy W2 from exact operand codes
        dyd = omx.roundtrip_rows(dy[tok])
        dh = b["dh"][sl]
        bdh = acc_band(dyd, wbound(w2[e].T))

        def parts(gg, uu, dd):
            sg = omoe.sigmoid(gg)
            s = gg * sg
            return dd * p * uu * sg * (1 + gg * (1 - sg)), dd * p * s, p * s * uu, dd * s * uu

        base = parts(g, u, dh)
        band = [np.zeros_like(t) for t in base]
        for gg in (lo[:, :I], hi[:, :I], g):
            for uu in (lo[:, I:], hi[:, I:], u):
                alt = parts(gg, uu, dh)
                for i in range(4):
                    band[i] = np.maximum(band[i], np.abs(alt[i] - base[i]))
        sg = omoe.sigmoid(g)
        band[0] += np.abs(p * u * sg * (1 + g * (1 - sg))) * bdh + ACT * np.abs(base[0])
        band[1] += np.abs(p * g * sg) * bdh + ACT * np.abs(base[1])
        band[2] += ACT * np.abs(base[2])
        band[3] += np.abs(g * sg * u) * bdh + ACT * np.abs(base[3])
        allow_dp[sl] = band[3].sum(axis=1)
        da = np.concatenate([base[0], base[1]], axis=1)
        bda = np.concatenate([band[0], band[1]], axis=1)
        # dgrad1: ambiguous row-wise da codes times |W1| (quantised along 2I)
        Dr = code_ambiguity(da, bda)
        allow_dx[sl] = Dr @ wbound(w1[e].T).T
        # wgrad2: |dy| (exact codes) times ambiguous h codes along tokens
        Dh = code_ambiguity_cols(base[2], band[2], [m])[0]
        dyc = omx.roundtrip_cols_grouped(dy[tok], [m])[0]
        aW2[e] = np.abs(dyc) @ Dh.T
        # wgrad1: ambiguous da codes along tokens times |x| (exact codes)
        Dc = code_ambiguity_cols(da, bda, [m])[0]
        xc = omx.roundtrip_cols_grouped(x[tok], [m])[0]
        aW1[e] = Dc @ np.abs(xc).T
    aX = allow_dx[f["slot_row"]].reshape(T, k, -1).sum(axis=1)
    dprob = np.zeros(R)
    dprob[f["perm"]] = allow_dp
    return {"dX": aX, "dW1": aW1, "dW2": aW2, "dprob": dprob.reshape(T, k)}


def bf16_ambiguity(v: np.ndarray, band: np.ndarray) -> np.ndarray:
    """max |bf16(any value in [v-band, v+band]) - bf16(v)| (rounding is
    monotone, so the ends of the band give it)."""
    ref = omoe.bf16_round(v)
    lo, hi = bf16_alternatives(v, band)
    return np.maximum(np.abs(lo - ref), np.abs(hi - ref))


def backward_allowance_bf16(f, b, x, w1, w2, dy, topk_idx):
    """Element-wise allowances for dX, dW1, dW2 and dprob of the BF16
    recipe's backward: the operands are exact bf16 values, and the tensors
    held in bf16 between the GEMMs (the saved A, da = [dg | du] and h) may
    round either way where their value is ambiguous."""
    E, I2, H = w1.shape
    I = I2 // 2
    T, k = topk_idx.shape
    R = f["perm"].size
    allow_dx = np.zeros((R, H))
    allow_dp = np.zeros(R)
    aW1 = np.zeros(w1.shape)
    aW2 = np.zeros(w2.shape)
    for e, sl in enumerate(_rows_by_expert(f["offsets"], E)):
        m = sl.stop - sl.start
        if m == 0:
            continue
        tok = f["tok"][sl]
        p = f["p"][sl][:, None]
        xg, dyg = x[tok], dy[tok]
        lo, hi = bf16_alternatives(f["A"][sl], acc_band(xg, w1[e]))
        a = f["saved"][sl]
        g, u = a[:, :I], a[:, I:]
        dh = b["dh"][sl]
        bdh = acc_band(dyg, w2[e].T)

        def parts(gg, uu, dd):
            sg = omoe.sigmoid(gg)
            s = gg * sg
            return dd * p * uu * sg * (1 + gg * (1 - sg)), dd * p * s, p * s * uu, dd * s * uu

        base = parts(g, u, dh)
        band = [np.zeros_like(t) for t in base]
        for gg in (lo[:, :I], hi[:, :I], g):
            for uu in (lo[:, I:], hi[:, I:], u):
                alt = parts(gg, uu, dh)
                for i in range(4):
                    band[i] = np.maximum(band[i], np.abs(alt[i] - base[i]))
        sg = omoe.sigmoid(g)
        band[0] += np.abs(p * u * sg * (1 + g * (1 - sg))) * bdh + ACT * np.abs(base[0])
        band[1] += np.abs(p * g * sg) * bdh + ACT * np.abs(base[1])
        band[2] += ACT * np.abs(base[2])
        band[3] += np.abs(g * sg * u) * bdh + ACT * np.abs(base[3])
        allow_dp[sl] = band[3].sum(axis=1)
        Dda = bf16_ambiguity(np.concatenate([base[0], base[1]], axis=1),
                             np.concatenate([band[0], band[1]], axis=1))
        Dh = bf16_ambiguity(base[2], band[2])
        allow_dx[sl] = Dda @ np.abs(w1[e])          # dgrad1: da W_gate_up
        aW2[e] = np.abs(dyg).T @ Dh                  # wgrad2: dy^T h
        aW1[e] = Dda.T @ np.abs(xg)                  # wgrad1: da^T x
    aX = allow_dx[f["slot_row"]].reshape(T, k, -1).sum(axis=1)
    dprob = np.zeros(R)
    dprob[f["perm"]] = allow_dp
    return {"dX": aX, "dW1": aW1, "dW2": aW2, "dprob": dprob.reshape(T, k)}


def backward_allowance_f8t(f, b, dy, topk_idx):
    """Element-wise allowances for dX, dW1, dW2 and dprob of the per-tensor
    FP8 recipe's backward (oracle/fp8tensor.py): as the BF16 recipe's, with
    the operands dequantised through their factors and, for da and h, the
    change of the per-tensor round trip (at the oracle's factors) over the
    bf16 values an ambiguous element may take."""
    from oracle import fp8tensor as ft
    E, I2, H = f["w1q"].shape
    I = I2 // 2
    T, k = topk_idx.shape
    R = f["perm"].size
    xd = ft.dequantize_tensor(f["xq"], f["s_x"])
    dyd = ft.dequantize_tensor(ft.quantize_tensor(dy, b["s_dy"]), b["s_dy"])
    s_da, s_hb = b["s_da"], b["s_hb"]

    def code_amb(v, band, s):
        q = lambda t: ft.dequantize_tensor(ft.quantize_tensor(t, s), s)
        ref = q(omoe.bf16_round(v))
        lo, hi = bf16_alternatives(v, band)
        return np.maximum(np.abs(q(lo) - ref), np.abs(q(hi) - ref))

    allow_dx = np.zeros((R, H))
    allow_dp = np.zeros(R)
    aW1 = np.zeros((E, I2, H))
    aW2 = np.zeros((E, H, I))
    for e, sl in enumerate(_rows_by_expert(f["offsets"], E)):
        if sl.stop == sl.start:
            continue
        tok = f["tok"][sl]
        p = f["p"][sl][:, None]
        w1d = ft.dequantize_tensor(f["w1q"][e], f["s_w1"][e])
        w2d = ft.dequantize_tensor(f["w2q"][e], f["s_w2"][e])
        xg, dyg = xd[tok], dyd[tok]
        lo, hi = bf16_alternatives(f["A"][sl], acc_band(xg, w1d))
        a = f["saved"][sl]
        g, u = a[:, :I], a[:, I:]
        dh = b["dh"][sl]
        bdh = acc_band(dyg, w2d.T)

        def parts(gg, uu, dd):
            sg = omoe.sigmoid(gg)
            s = gg * sg
            return dd * p * uu * sg * (1 + gg * (1 - sg)), dd * p * s, p * s * uu, dd * s * uu

        base = parts(g, u, dh)
        band = [np.zeros_like(t) for t in base]
        for gg in (lo[:, :I], hi[:, :I], g):
            for uu in (lo[:, I:], hi[:, I:], u):
                alt = parts(gg, uu, dh)
                for i in range(4):
                    band[i] = np.maximum(band[i], np.abs(alt[i] - base[i]))
        sg = omoe.sigmoid(g)
        band[0] += np.abs(p * u * sg * (1 + g * (1 - sg))) * bdh + ACT * np.abs(base[0])
        band[1] += np.abs(p * g * sg) * bdh + ACT * np.abs(base[1])
        band[2] += ACT * np.abs(base[2])
        band[3] += np.abs(g * sg * u) * bdh + ACT * np.abs(base[3])
        allow_dp[sl] = band[3].sum(axis=1)
        Dda = code_amb(np.concatenate([base[0], base[1]], axis=1), np.concatenate([band[0], band[1]], axis=1), s_da)
        Dh = code_amb(base[2], band[2], s_hb)
        allow_dx[sl] = Dda @ np.abs(w1d)             # dgrad1: da W_gate_up
        aW2[e] = np.abs(dyg).T @ Dh                   # wgrad2: dy^T h
        aW1[e] = Dda.T @ np.abs(xg)                   # wgrad1: da^T x
    aX = allow_dx[f["slot_row"]].reshape(T, k, -1).sum(axis=1)
    dprob = np.zeros(R)
    dprob[f["perm"]] = allow_dp
    return {"dX": aX, "dW1": aW1, "dW2": aW2, "dprob": dprob.reshape(T, k)}


def within(gpu, ref, tol, allow, bf16_out=True):
    """max over elements of (|gpu - ref| - allow) / rms(ref), to compare
    with tol.  For bf16 outputs the allowance also holds the output's own
    rounding, half a bf16 ulp <= 2^-8 |ref|: the oracle's reference is the
    unrounded float64 value."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    if bf16_out:
        allow = allow + 2.0 ** -8 * np.abs(ref)
    excess = np.abs(gpu - ref) - allow
    return float(np.max(excess) / rms)
