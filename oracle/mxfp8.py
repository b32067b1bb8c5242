"""MXFP8 codec of the oracle (float64, numpy).  Test infrastructure only.

The pages fix one fact about the format ("Efficient MoE Training for
Biological Foundation Models", Challenge 2): values are 8-bit and every
block of 32 consecutive values shares one scaling factor.  The rest is the
plainest reading consistent with that and with Blackwell's block-scaled
tensor-core operands:

* element type E4M3 (bias 7, 3 mantissa bits, subnormals down to 2^-9,
  largest finite 448, no infinity, 0x7F/0xFF are NaN);
* scale type E8M0: a bare power of two 2^(b-127), b = 0xFF is NaN;
* a block is 32 consecutive values along the contraction (K) axis of the
  GEMM that consumes it, starting at index 0;
* scale exponent s = the smallest power of two with amax / 2^s <= 448.  With
  amax = m * 2^e, m in [1, 2): s = e - 8, plus 1 when m > 1.75.  s is
  clamped to [-127, 127]; an all-zero block gets s = -127; a block holding a
  NaN or an infinity gets the NaN scale byte 0xFF and NaN elements;
* element code = E4M3(v * 2^-s), round to nearest, ties to even mantissa,
  saturating to +-448 (never reached with the rule above).
"""
from __future__ import annotations

import numpy as np

BLOCK = 32
E4M3_MAX = 448.0
SCALE_NAN = 0xFF
CODE_NAN = 0x7F


def _e4m3_value(code: int) -> float:
    """Value of one E4M3 code from the format definition."""
    sign = -1.0 if code & 0x80 else 1.0
    ex = (code >> 3) & 0xF
    man = code & 0x7
    if ex == 0xF and man == 0x7:
        return float("nan")
    if ex == 0:
        return sign * man * 2.0 ** -9
    return sign * (1.0 + man / 8.0) * 2.0 ** (ex - 7)


E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


# Non-negative finite E4M3 values in code order (codes 0x00..0x7E are
# increasing) and the midpoints between neighbours.
_POS_VALUES = E4M3_TABLE[:0x7F]
_MIDPOINTS = 0.5 * (_POS_VALUES[:-1] + _POS_VALUES[1:])


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """float64 -> E4M3 codes: the nearest finite E4M3 value, ties to the even
    code (even mantissa), saturating at +-448 (values above 448 round to the
    largest code).  NaN (and infinity, which the scale rule never produces
    here) -> 0x7F with the sign bit of the input."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    bad = ~np.isfinite(a)
    a = np.where(bad, 0.0, a)
    # number of midpoints strictly below a = index of the nearest value,
    # except at an exact midpoint, where it is the lower neighbour
    code = np.searchsorted(_MIDPOINTS, a, side="left")
    tie = (code < _MIDPOINTS.size) & (a == _MIDPOINTS[np.minimum(code, _MIDPOINTS.size - 1)])
    code = code + (tie & (code % 2 == 1))
    code = np.where(bad, CODE_NAN, code)
    code = code | (np.signbit(v).astype(np.int64) << 7)
    return code.astype(np.uint8)


def scale_exponent(amax: np.ndarray) -> np.ndarray:
    """Block amax -> E8M0 scale byte (see module docstring)."""
    amax = np.asarray(amax, dtype=np.float64)
    bad = ~np.isfinite(amax)
    am = np.where(bad, 0.0, amax)
    f, ex = np.frexp(am)                     # am = f * 2^ex, f in [0.5, 1)
    m, e = 2.0 * f, ex - 1                   # am = m * 2^e, m in [1, 2)
    s = e - 8 + (m > 1.75).astype(np.int64)
    s = np.where(am == 0.0, -127, s)
    s = np.clip(s, -127, 127)
    b = (s + 127).astype(np.int64)
    return np.where(bad, SCALE_NAN, b).astype(np.uint8)


def scale_value(sbytes: np.ndarray) -> np.ndarray:
    sb = np.asarray(sbytes, dtype=np.int64)
    v = np.ldexp(1.0, sb - 127)
    return np.where(sb == SCALE_NAN, np.nan, v)


def quantize_rows(x: np.ndarray):
    """Quantise a 2-D array along its last axis (the GEMM's K axis), in
    blocks of 32 starting at column 0.  Returns (codes uint8 [M, K],
    scale bytes uint8 [M, K/32])."""
    x = np.asarray(x, dtype=np.float64)
    M, K = x.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 32")
    blk = x.reshape(M, K // BLOCK, BLOCK)
    with np.errstate(invalid="ignore"):
        amax = np.max(np.abs(blk), axis=2)
    has_nan = np.isnan(blk).any(axis=2)
    amax = np.where(has_nan, np.nan, amax)
    sb = scale_exponent(amax)
    inv = np.ldexp(1.0, 127 - sb.astype(np.int64))        # 2^-s, exact
    inv = np.where(sb == SCALE_NAN, np.nan, inv)
    codes = e4m3_encode(blk * inv[:, :, None]).reshape(M, K)
    return codes, sb


def dequantize_rows(codes: np.ndarray, sbytes: np.ndarray) -> np.ndarray:
    """Inverse of quantize_rows: E4M3 value times 2^s, float64."""
    M, K = codes.shape
    v = e4m3_decode(codes).reshape(M, K // BLOCK, BLOCK)
    return (v * scale_value(sbytes)[:, :, None]).reshape(M, K)


def roundtrip_rows(x: np.ndarray) -> np.ndarray:
    """dequantize(quantize(x)) along the last axis."""
    return dequantize_rows(*quantize_rows(x))


def quantize_cols_grouped(x: np.ndarray, group_sizes):
    """Quantise along axis 0 (tokens) inside each group of consecutive rows.

    Reading taken for ragged groups (the pages are silent): 32-row blocks
    start at each group's first row; a partial last block is padded with
    zeros, which change neither its amax nor any sum; an empty group has no
    blocks.  Returns a list, one entry per group, of (codes uint8
    [N, Mpad_g], scale bytes uint8 [N, Mpad_g/32]) for the TRANSPOSED group
    x_g^T (so the block axis is the last one), Mpad_g = ceil(M_g/32)*32.
    """
    x = np.asarray(x, dtype=np.float64)
    out, r0 = [], 0
    for m in group_sizes:
        m = int(m)
        mp = -(-m // BLOCK) * BLOCK
        g = np.zeros((x.shape[1], mp), dtype=np.float64)
        g[:, :m] = x[r0:r0 + m].T
        out.append(quantize_rows(g) if mp else (np.zeros((x.shape[1], 0), np.uint8),
                                                np.zeros((x.shape[1], 0), np.uint8)))
        r0 += m
    return out


def roundtrip_cols_grouped(x: np.ndarray, group_sizes) -> list:
    """Per group g: dequantised x_g^T [N, M_g] (padding dropped)."""
    res = []
    for (c, s), m in zip(quantize_cols_grouped(x, group_sizes), group_sizes):
        res.append(dequantize_rows(c, s)[:, :int(m)] if c.shape[1] else np.zeros((x.shape[1], 0)))
    return res
