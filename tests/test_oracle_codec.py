"""Pins of the oracle's MXFP8 codec against things other than itself:
brute force over every code, library casts (ml_dtypes, torch), the format
fixtures in tests/golden/, and the minimality property of the scale rule.
MXFP8 per "Efficient MoE Training for Biological Foundation Models",
Challenge 2 (8-bit values, one scale per 32 consecutive values)."""
import os

import numpy as np
import pytest

from oracle import mxfp8

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _all_bf16_values():
    bits = np.arange(65536, dtype=np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):  # the NaN patterns (dropped below) signal on the cast
        v = bits.view(np.float32).astype(np.float64)
    return v[np.isfinite(v)]


def _brute_encode(v):
    """Nearest finite E4M3 code by exhaustive search; ties to the even
    mantissa; beyond 448 saturate."""
    codes = np.array([c for c in range(256) if np.isfinite(mxfp8.E4M3_TABLE[c])])
    vals = mxfp8.E4M3_TABLE[codes]
    out = np.empty(v.shape, np.uint8)
    for i, x in enumerate(v):
        if abs(x) > 448.0:
            c = 0x7E | (0x80 if x < 0 else 0)
        else:
            d = np.abs(vals - x)
            best = np.flatnonzero(d == d.min())
            # same-sign candidates only (a signed zero pair is a tie of equal value)
            best = [b for b in codes[best] if (b >> 7) == (1 if np.signbit(x) else 0)] or list(codes[best])
            if len(best) > 1:
                best = [b for b in best if (b & 1) == 0]
            c = best[0]
        out[i] = c
    return out


def test_decode_table_format():
    t = mxfp8.E4M3_TABLE
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert np.sum(np.isnan(t)) == 2
    assert t[0x7E] == 448.0 and t[0x01] == 2.0 ** -9 and t[0x38] == 1.0
    # monotone over positive codes, antisymmetric sign bit
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0)
    assert np.array_equal(t[0x80:0xFF], -t[0x00:0x7F])


def test_golden_e4m3_fixtures():
    with open(os.path.join(GOLDEN, "e4m3_format.txt")) as fh:
        rows = [ln.split() for ln in fh if ln.strip() and not ln.startswith("#")]
    v = np.array([float(r[0]) for r in rows])
    want = np.array([int(r[1], 16) for r in rows], np.uint8)
    assert np.array_equal(mxfp8.e4m3_encode(v), want)


def test_golden_scale_fixtures():
    with open(os.path.join(GOLDEN, "e8m0_scale.txt")) as fh:
        rows = [ln.split() for ln in fh if ln.strip() and not ln.startswith("#")]
    amax = np.array([float(r[0]) for r in rows])
    want = np.array([int(r[1]) for r in rows], np.uint8)
    assert np.array_equal(mxfp8.scale_exponent(amax), want)


@pytest.mark.parametrize("shift", [-12, -9, -6, -3, 0, 3, 6, 8, 9])
def test_encode_matches_brute_force_every_bf16(shift):
    """Every finite bf16 pattern, scaled by 2^shift into and around the E4M3
    range (subnormals, normals, saturation), against exhaustive search.
    Sampled to keep the CPU suite fast: all patterns whose magnitude lands
    in [2^-12, 2^10] after scaling, which covers every E4M3 binade."""
    v = _all_bf16_values() * 2.0 ** shift
    a = np.abs(v)
    v = v[(a == 0) | ((a >= 2.0 ** -12) & (a <= 2.0 ** 10))]
    got = mxfp8.e4m3_encode(v)
    want = _brute_encode(v)
    assert np.array_equal(got, want)


def test_encode_matches_library_casts():
    import ml_dtypes
    import torch
    v = _all_bf16_values()
    v = v[np.abs(v) <= 448.0]
    f32 = v.astype(np.float32)
    ml = f32.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    th = torch.from_numpy(f32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = mxfp8.e4m3_encode(v)
    assert np.array_equal(got, ml)
    assert np.array_equal(got, th)


def test_scale_rule_is_smallest_power_of_two():
    """s must be the smallest integer with amax / 2^s <= 448 (search, not
    the closed form), clamped to [-127, 127]."""
    rng = np.random.default_rng(1)
    amax = np.concatenate([
        np.ldexp(rng.uniform(1, 2, 4000), rng.integers(-140, 127, 4000)),
        np.ldexp(np.array([1.75, 1.75 + 2 ** -20, 1.0, 1.5, 1.9999]), 3),
        _all_bf16_values()[::97],
    ])
    amax = np.abs(amax)
    got = mxfp8.scale_exponent(amax).astype(int) - 127
    for a, s in zip(amax, got):
        if a == 0:
            assert s == -127
            continue
        cand = [t for t in range(-200, 200) if a <= 448.0 * 2.0 ** t][0]
        assert s == min(max(cand, -127), 127), (a, s, cand)


def test_scale_rule_matches_torch_float8_cast_saturation_bound():
    """With the chosen scale no element of a block exceeds 448 after
    scaling, and halving the scale would overflow the block maximum."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 256)) * np.ldexp(1.0, rng.integers(-20, 20, (64, 1)))
    c, s = mxfp8.quantize_rows(x)
    sc = mxfp8.scale_value(s)
    blk = np.abs(x).reshape(64, 8, 32).max(axis=2)
    assert np.all(blk / sc <= 448.0)
    assert np.all(blk / (sc / 2) > 448.0)


def test_quantize_roundtrip_error_bound():
    """Round trip error is at most half an E4M3 ulp of the scaled value:
    2^-4 relative for normals, 2^-10 * 2^s absolute for subnormals."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((32, 512)) * 3.0
    c, s = mxfp8.quantize_rows(x)
    d = mxfp8.dequantize_rows(c, s)
    sc = np.repeat(mxfp8.scale_value(s), 32, axis=1)
    y = np.abs(x) / sc
    bound = np.where(y >= 2.0 ** -6, y * 2.0 ** -4, 2.0 ** -10) * sc
    assert np.all(np.abs(d - x) <= bound * (1 + 1e-12))
    assert np.all(np.abs(mxfp8.e4m3_decode(c)) <= 448.0)


def test_scales_are_powers_of_two_and_codes_bounded():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((16, 2880))
    c, s = mxfp8.quantize_rows(x)
    assert c.shape == (16, 2880) and s.shape == (16, 90)
    assert np.all(s != 0xFF)
    v = mxfp8.scale_value(s)
    assert np.all(np.log2(v) == np.round(np.log2(v)))
    assert np.all(np.isfinite(mxfp8.e4m3_decode(c)))


def test_zero_and_nan_blocks():
    x = np.zeros((2, 64))
    x[1, 40] = np.nan
    c, s = mxfp8.quantize_rows(x)
    assert s[0, 0] == 0 and s[0, 1] == 0 and np.all(c[0] == 0)
    assert s[1, 0] == 0 and s[1, 1] == 0xFF
    assert np.all((c[1, 32:] & 0x7F) == 0x7F)


def test_exactly_representable_values_roundtrip_exactly():
    """Values that are E4M3 codes times a common power of two survive."""
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 0x7F, (8, 64)).astype(np.uint8)
    codes[:, ::32] = 0x7E                         # block max 448 -> s = 0
    v = mxfp8.e4m3_decode(codes) * 2.0 ** -5
    c, s = mxfp8.quantize_rows(v)
    assert np.all(s == 127 - 5)
    assert np.array_equal(mxfp8.dequantize_rows(c, s), v)


def test_cols_grouped_blocks_start_at_group_rows():
    """Column-wise quantisation along tokens restarts at each group; a
    partial last block is zero padded and an empty group has no blocks."""
    rng = np.random.default_rng(6)
    x = rng.standard_normal((70, 8))
    groups = [33, 0, 37]
    q = mxfp8.quantize_cols_grouped(x, groups)
    assert q[0][0].shape == (8, 64) and q[1][0].shape == (8, 0) and q[2][0].shape == (8, 64)
    # group 2 equals quantising its own rows transposed and zero padded
    g = np.zeros((8, 64))
    g[:, :37] = x[33:].T
    c, s = mxfp8.quantize_rows(g)
    assert np.array_equal(q[2][0], c) and np.array_equal(q[2][1], s)
    # padding codes are zero
    assert np.all(q[0][0][:, 33:] == 0)
