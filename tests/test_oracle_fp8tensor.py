"""Pins of the per-tensor FP8 oracle (oracle/fp8tensor.py) against what the
format definitions and the arithmetic fix, independently of its code."""
from fractions import Fraction
import struct

import numpy as np
import pytest

from oracle import fp8tensor as ft
from oracle import moe as omoe
from oracle.mxfp8 import E4M3_TABLE
from mxfp8_grouped_gemm_x32_b200.workloads import bf16_bits_to_f32


def _f32(x: float) -> float:
    return struct.unpack("<f", struct.pack("<f", x))[0]


def _f32_neighbours(r: float):
    b = struct.unpack("<I", struct.pack("<f", r))[0]
    return [struct.unpack("<f", struct.pack("<I", b + d))[0] for d in (-1, 1)]


def test_scale_is_448_over_amax_rounded_to_float32():
    """The factor is the float32 nearest to 448 / amax (checked against the
    exact rational value), the largest finite float32 where that overflows,
    1 for an all-zero or non-finite tensor."""
    assert ft.tensor_scale(np.array([0.0, -448.0, 3.0])) == np.float32(1.0)
    assert ft.tensor_scale(np.array([1.0, -0.5])) == np.float32(448.0)
    assert ft.tensor_scale(np.zeros(5)) == np.float32(1.0)
    assert ft.tensor_scale(np.array([1.0, np.nan])) == np.float32(1.0)
    rng = np.random.default_rng(0)
    bits = rng.integers(0x0080, 0x7F80, size=2000).astype(np.uint16)          # finite positive bf16
    vals = bf16_bits_to_f32(bits).astype(np.float64)
    fmax = float(np.finfo(np.float32).max)
    for a in vals:
        r = float(ft.tensor_scale(np.array([a, -a / 2])))
        exact = Fraction(448) / Fraction(a)
        if exact > Fraction(fmax) + Fraction(2) ** 103:     # past the float32 range (and its rounding half-ulp)
            assert r == fmax
            continue
        err = abs(Fraction(r) - exact)
        assert all(err <= abs(Fraction(n) - exact) for n in _f32_neighbours(r))


def _nearest_e4m3(v: float) -> int:
    """Brute force over the 254 finite codes: nearest value, ties to the even
    code, saturating at +-448."""
    a = min(abs(v), 448.0)
    best = None
    for c in range(0x7F):
        d = abs(E4M3_TABLE[c] - a)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return best[1] | (0x80 if np.signbit(v) else 0)


def test_code_is_nearest_e4m3_of_the_float32_product():
    """code = nearest E4M3 of float32(v * scale): the product is rounded to
    float32 first (a product that lands on an E4M3 midpoint only after that
    rounding decides the tie differently from the exact product)."""
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 0x10000, size=3000).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]                                  # finite values only
    v = bf16_bits_to_f32(bits).astype(np.float64)
    s = np.float32(448.0) / np.float32(np.max(np.abs(v)))
    codes = ft.quantize_tensor(v, s)
    for vi, ci in zip(v[:600], codes[:600]):
        prod = _f32(float(Fraction(vi) * Fraction(float(s))))             # exact product rounded to float32
        assert ci == _nearest_e4m3(prod)
    # a case where the rounding order matters: the exact product sits just
    # above an E4M3 midpoint (1.0625 between 1.0 and 1.125) and rounds down to
    # it in float32, where the tie goes to the even code 1.0
    v1, s1 = 1.0625 + 2.0 ** -23, np.float32(1.0 - 2.0 ** -24)
    exact = Fraction(v1) * Fraction(float(s1))
    assert Fraction(1.0625) < exact < Fraction(1.0625) + Fraction(2) ** -24
    assert float(np.float32(v1) * s1) == 1.0625
    assert ft.quantize_tensor(np.array([v1]), s1)[0] == 0x38            # 1.0, not 1.125


def _case(T=48, H=64, I=32, E=3, k=2, seed=0):
    rng = np.random.default_rng(seed)
    bf = lambda a: bf16_bits_to_f32(omoe.bf16_bits(a)).astype(np.float64)
    x = bf(rng.standard_normal((T, H)))
    w1 = bf(rng.standard_normal((E, 2 * I, H)) / np.sqrt(H))
    w2 = bf(rng.standard_normal((E, H, I)) / np.sqrt(I))
    logits = rng.standard_normal((T, E))
    idx = np.argsort(-logits, axis=1, kind="stable")[:, :k].astype(np.int32)
    p = np.exp(np.take_along_axis(logits, idx, 1))
    return x, w1, w2, idx, (p / p.sum(1, keepdims=True)).astype(np.float32)


def test_identity_expert_closed_form():
    """W_gate_up = identity, W_down = [I; 0], p = 1, x of E4M3 values with
    amax 448: every factor but h's is exact, so out = [Q(h), 0] with
    h = bf16(silu(x1) * x2) and Q the round trip through the factor
    448 / amax(h) -- written out here from the definitions."""
    I = 32
    H = 2 * I
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 0x7F, size=(16, H))
    x = E4M3_TABLE[codes] * np.where(rng.random((16, H)) < 0.5, -1.0, 1.0)
    x[0, 0] = 448.0
    w1 = np.eye(2 * I)[None]
    w2 = np.concatenate([np.eye(I), np.zeros((I, I))])[None]
    idx = np.zeros((16, 1), np.int32)
    prob = np.ones((16, 1), np.float32)
    f = ft.forward(x, w1, w2, idx, prob)
    assert f["s_x"] == np.float32(1.0) and np.all(f["s_w1"] == np.float32(448.0))
    x1, x2 = x[:, :I], x[:, I:]
    h = bf16_bits_to_f32(omoe.bf16_bits(x1 / (1.0 + np.exp(-x1)) * x2)).astype(np.float64)
    amax = np.max(np.abs(h))
    s_h = _f32(float(Fraction(448) / Fraction(amax)))
    want = np.array([[E4M3_TABLE[_nearest_e4m3(_f32(float(Fraction(v) * Fraction(s_h))))] for v in row]
                     for row in h]) / s_h
    got = f["out"]
    assert np.array_equal(got[:, :I], want) and np.all(got[:, I:] == 0)


def test_gate_up_result_scales_with_the_input():
    """x -> 2^5 x: the factor divides by exactly 2^5, the codes are the same
    and A is multiplied by exactly 2^5 (a dropped or doubled factor breaks
    this)."""
    x, w1, w2, idx, p = _case()
    a = ft.forward(x, w1, w2, idx, p)
    b = ft.forward(x * 32.0, w1, w2, idx, p)
    assert b["s_x"] * np.float32(32.0) == a["s_x"]
    assert np.array_equal(a["xq"], b["xq"])
    assert np.array_equal(b["A"], 32.0 * a["A"])


def test_close_to_the_unquantised_layer():
    """FP8 rounding error only: out within 10 % of the rms of the exact
    layer in rms (E4M3 keeps 3 mantissa bits; MXFP8 gives about the same on
    these inputs) and no element off by more than the rms."""
    x, w1, w2, idx, p = _case(seed=5)
    q = ft.forward(x, w1, w2, idx, p)["out"]
    ref = omoe.forward(x, w1, w2, idx, p, quantize=False)["out"]
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.sqrt(np.mean((q - ref) ** 2)) <= 0.1 * rms
    assert np.max(np.abs(q - ref)) <= rms


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------

def _q_brute(v: np.ndarray) -> np.ndarray:
    """Per-tensor round trip written out from the definitions: factor = the
    float32 nearest to 448 / amax (exact rational), code = nearest E4M3 of
    the float32 product, value = code / factor."""
    amax = float(np.max(np.abs(v)))
    s = _f32(float(Fraction(448) / Fraction(amax)))
    flat = [E4M3_TABLE[_nearest_e4m3(_f32(float(Fraction(x) * Fraction(s))))]    # code carries the sign
            for x in np.asarray(v, np.float64).reshape(-1)]
    return np.array(flat).reshape(np.shape(v)) / s


def test_backward_identity_expert_closed_form():
    """W_gate_up = identity, W_down = [I; 0], p = 1, x and dY of E4M3 values
    with |max| 448: x, the weights and dY quantise exactly, so dh = dY[:, :I]
    and dX = Q(da), dW_gate_up = Q(da)^T x, dW_down = dY^T Q(h), dprob =
    sum dh*silu(g)*u, with da = bf16([dg, du]), h = bf16(silu(g)*u) and Q the
    round trip through each tensor's factor -- all written out here from the
    definitions (brute-force E4M3, exact-rational factors)."""
    I = 32
    H = 2 * I
    T = 16
    rng = np.random.default_rng(11)
    sign = lambda shape: np.where(rng.random(shape) < 0.5, -1.0, 1.0)
    x = E4M3_TABLE[rng.integers(0, 0x7F, size=(T, H))] * sign((T, H)) / 64.0
    x[0, 0] = 448.0 / 64.0                                       # amax 7 -> factor 64, still exact
    dy = E4M3_TABLE[rng.integers(0, 0x7F, size=(T, H))] * sign((T, H))
    dy[1, 3] = -448.0
    w1 = np.eye(2 * I)[None]
    w2 = np.concatenate([np.eye(I), np.zeros((I, I))])[None]
    idx = np.zeros((T, 1), np.int32)
    prob = np.ones((T, 1), np.float32)
    f = ft.forward(x, w1, w2, idx, prob)
    assert f["s_x"] == np.float32(64.0)
    b = ft.backward(f, dy, prob)
    assert b["s_dy"] == np.float32(1.0)
    g, u = omoe.bf16_round(x[:, :I]), omoe.bf16_round(x[:, I:])
    sg = 1.0 / (1.0 + np.exp(-g))
    dh = dy[:, :I]
    da = omoe.bf16_round(np.concatenate([dh * u * sg * (1.0 + g * (1.0 - sg)), dh * g * sg], axis=1))
    hb = omoe.bf16_round(g * sg * u)
    qda, qh = _q_brute(da), _q_brute(hb)
    assert np.array_equal(b["dX"], qda)
    assert np.allclose(b["dW1"][0], qda.T @ x, rtol=1e-12, atol=1e-12)
    assert np.allclose(b["dW2"][0], dy.T @ qh, rtol=1e-12, atol=1e-12)
    assert np.allclose(b["dprob_f64"][:, 0], np.sum(dh * g * sg * u, axis=1), rtol=1e-12, atol=1e-12)


def test_backward_scales_exactly_with_dy():
    """dY -> 2^5 dY: its factor divides by exactly 2^5 and every gradient is
    multiplied by exactly 2^5 (dh, da and their codes scale through; h does
    not depend on dY) -- a dropped, doubled or misplaced factor breaks this."""
    x, w1, w2, idx, p = _case(seed=7)
    rng = np.random.default_rng(8)
    dy = bf16_bits_to_f32(omoe.bf16_bits(rng.standard_normal(x.shape))).astype(np.float64)
    f = ft.forward(x, w1, w2, idx, p)
    a = ft.backward(f, dy, p)
    b = ft.backward(f, dy * 32.0, p)
    assert b["s_dy"] * np.float32(32.0) == a["s_dy"] and b["s_da"] * np.float32(32.0) == a["s_da"]
    assert b["s_hb"] == a["s_hb"]
    for key in ("dX", "dW1", "dW2", "dprob_f64"):
        assert np.array_equal(b[key], 32.0 * a[key]), key


def test_backward_close_to_the_unquantised_layer():
    """FP8 rounding error only: every gradient within 12 % of the rms of the
    exact layer's gradient in rms (a transposed operand, a wrong row or a
    dropped term gives errors of the order of the rms itself)."""
    x, w1, w2, idx, p = _case(seed=9)
    rng = np.random.default_rng(10)
    dy = bf16_bits_to_f32(omoe.bf16_bits(rng.standard_normal(x.shape))).astype(np.float64)
    q = ft.backward(ft.forward(x, w1, w2, idx, p), dy, p)
    fe = omoe.forward(x, w1, w2, idx, p, quantize=False, round_saved=False)
    ref = omoe.backward(fe, x, w1, w2, p, dy, quantize=False)
    for key, rk in (("dX", "dX"), ("dW1", "dW1"), ("dW2", "dW2"), ("dprob_f64", "dprob_f64")):
        rms = np.sqrt(np.mean(ref[rk] ** 2))
        assert np.sqrt(np.mean((q[key] - ref[rk]) ** 2)) <= 0.12 * rms, key
