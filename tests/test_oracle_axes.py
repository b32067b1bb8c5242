"""Pins of the oracle's quantisation axes (test infrastructure, CPU only).

"Efficient MoE Training for Biological Foundation Models", Challenge 2 and
Challenge 3: every low-precision GEMM operand carries one scale per 32
consecutive values along that GEMM's contraction axis.  The oracle's reading
(one block axis per operand, forward and backward) is pinned here by inputs
that make the wrong axis fail loudly: an operand whose rows (or columns) are
scaled by powers of two spread over 2^21 inside every run of 32 keeps each
row (column) accurate to a few per cent when its blocks run along the scaled
axis's complement, and flushes the small rows (columns) to zero -- an error
near 100% -- when they run the other way.  Each check compares the quantised
oracle with its own unquantised mode (itself pinned by the per-expert loop
and finite differences in test_oracle_moe.py), one row or column at a time.

A planted mistake (the oracle's quantisers swapped to the other axis, on the
CPU) must make the matching pins fail; that is tested too.
"""
import types

import numpy as np

from oracle import moe, mxfp8

T, H, I = 64, 64, 64          # one expert, top-1: square operands, two 32-blocks per axis
BAR = 0.3                     # per-row relative error bound (correct axes: at most 0.12); the wrong axis gives ~1


def _spread(n):
    """Powers of two 2^0 .. 2^21, repeating every 8: every 32-run spans 2^21."""
    return 2.0 ** (3 * (np.arange(n) % 8))


def _rel_rows(q, ref):
    with np.errstate(invalid="ignore", divide="ignore"):
        return np.linalg.norm(q - ref, axis=1) / np.linalg.norm(ref, axis=1)


def _rel_cols(q, ref):
    return _rel_rows(q.T, ref.T)


def _inputs(seed, x_rows=None, x_cols=None, w1_rows=None, w1_up_rows=None, w2_rows=None, w2_cols=None,
            dy_rows=None, dy_cols=None):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H))
    w1 = rng.standard_normal((1, 2 * I, H)) / np.sqrt(H)
    w2 = rng.standard_normal((1, H, I)) / np.sqrt(I)
    dy = rng.standard_normal((T, H))
    if x_rows is not None:
        x *= x_rows[:, None]
    if x_cols is not None:
        x *= x_cols[None, :]
    if w1_rows is not None:
        w1[0] *= w1_rows[:, None]
    if w1_up_rows is not None:
        w1[0, I:] *= w1_up_rows[:, None]
    if w2_rows is not None:
        w2[0] *= w2_rows[:, None]
    if w2_cols is not None:
        w2[0] *= w2_cols[None, :]
    if dy_rows is not None:
        dy *= dy_rows[:, None]
    if dy_cols is not None:
        dy *= dy_cols[None, :]
    idx = np.zeros((T, 1), np.int32)
    prob = rng.uniform(0.3, 1.0, (T, 1)).astype(np.float32)
    return x, w1, w2, dy, idx, prob


def _run(inp, bwd=True):
    with np.errstate(over="ignore"):      # exp(-z) of the widely scaled gates overflows to inf: silu -> 0
        return _run_layer(inp, bwd)


def _run_layer(inp, bwd):
    x, w1, w2, dy, idx, prob = inp
    fq = moe.forward(x, w1, w2, idx, prob)
    fr = moe.forward(x, w1, w2, idx, prob, quantize=False, round_saved=False)
    if not bwd:
        return fq, fr, None, None
    # both backward passes start from the same saved activation, so that only
    # the backward's own quantisation differs between them
    fr["saved"] = fq["saved"]
    bq = moe.backward(fq, x, w1, w2, prob, dy)
    br = moe.backward(fr, x, w1, w2, prob, dy, quantize=False)
    return fq, fr, bq, br


# Each check: operand and axis pinned -> per-row (or per-column) relative error.
def _forward_checks():
    s = _spread
    out = {}
    fq, fr, _, _ = _run(_inputs(1, x_rows=s(T)), bwd=False)
    out["x, h along features"] = _rel_rows(fq["out"], fr["out"])     # token-scaled x (and so h)
    fq, fr, _, _ = _run(_inputs(2, w1_rows=s(2 * I)), bwd=False)
    out["W_gate_up along H"] = _rel_cols(fq["A"], fr["A"])           # A's columns follow W_gate_up's rows
    fq, fr, _, _ = _run(_inputs(3, w2_rows=s(H)), bwd=False)
    out["W_down along I"] = _rel_cols(fq["out"], fr["out"])          # out's columns follow W_down's rows
    return out


def _backward_checks():
    s = _spread
    out = {}
    _, _, bq, br = _run(_inputs(4, dy_rows=s(T)))
    out["dgrad2: dy along H"] = _rel_rows(bq["dh"], br["dh"])
    out["dgrad1: da along 2I"] = _rel_rows(bq["dx_rows"], br["dx_rows"])
    _, _, bq, br = _run(_inputs(5, dy_cols=s(H)))
    out["wgrad2: dy along tokens"] = _rel_rows(bq["dW2"][0], br["dW2"][0])
    _, _, bq, br = _run(_inputs(6, w1_up_rows=s(I)))
    out["wgrad2: h along tokens"] = _rel_cols(bq["dW2"][0], br["dW2"][0])
    _, _, bq, br = _run(_inputs(7, x_cols=s(H)))
    out["wgrad1: x along tokens"] = _rel_cols(bq["dW1"][0], br["dW1"][0])
    _, _, bq, br = _run(_inputs(8, w2_cols=s(I)))
    out["wgrad1: da along tokens"] = _rel_rows(bq["dW1"][0], br["dW1"][0])
    return out


def test_forward_quantisation_axes():
    for name, err in _forward_checks().items():
        assert np.isfinite(err).all() and err.max() <= BAR, (name, err.max())


def test_backward_quantisation_axes():
    for name, err in _backward_checks().items():
        assert np.isfinite(err).all() and err.max() <= BAR, (name, err.max())


# ---- planted mistakes (on the CPU, in the oracle) --------------------------

def _rows_along_axis0(v):
    return mxfp8.roundtrip_rows(np.asarray(v).T).T


def _cols_along_features(x, group_sizes):
    """The wgrad operands quantised along features instead of tokens."""
    res, r0 = [], 0
    for m in group_sizes:
        res.append(mxfp8.roundtrip_rows(np.asarray(x)[r0:r0 + int(m)]).T)
        r0 += int(m)
    return res


def _failing(checks):
    return {name for name, err in checks.items() if not (np.isfinite(err).all() and err.max() <= BAR)}


def test_planted_transposed_dgrad_and_weight_axes_are_caught(monkeypatch):
    # every roundtrip_rows operand (weights, dgrad operands) quantised along the other axis
    proxy = types.SimpleNamespace(**{n: getattr(mxfp8, n) for n in dir(mxfp8) if not n.startswith("__")})
    proxy.roundtrip_rows = _rows_along_axis0
    monkeypatch.setattr(moe, "mxfp8", proxy)
    assert {"W_gate_up along H", "W_down along I"} <= _failing(_forward_checks())
    assert {"dgrad2: dy along H", "dgrad1: da along 2I"} <= _failing(_backward_checks())


def test_planted_wgrad_along_features_is_caught(monkeypatch):
    proxy = types.SimpleNamespace(**{n: getattr(mxfp8, n) for n in dir(mxfp8) if not n.startswith("__")})
    proxy.roundtrip_cols_grouped = _cols_along_features
    monkeypatch.setattr(moe, "mxfp8", proxy)
    assert _failing(_backward_checks()) == {"wgrad2: dy along tokens", "wgrad2: h along tokens",
                                            "wgrad1: x along tokens", "wgrad1: da along tokens"}


def test_planted_activation_axis_is_caught(monkeypatch):
    # x and h (quantised with quantize_rows / dequantize_rows in the forward)
    # along tokens instead of features; the operands are square, so the
    # transposed codes and scales fit the same arrays
    proxy = types.SimpleNamespace(**{n: getattr(mxfp8, n) for n in dir(mxfp8) if not n.startswith("__")})
    proxy.quantize_rows = lambda v: mxfp8.quantize_rows(np.asarray(v).T)
    proxy.dequantize_rows = lambda c, s: mxfp8.dequantize_rows(c, s).T
    monkeypatch.setattr(moe, "mxfp8", proxy)
    assert "x, h along features" in _failing(_forward_checks())
