"""Pins of the oracle's MoE layer against things other than itself.

* P2: an independent restatement of the per-expert loop of "Efficient MoE
  Training for Biological Foundation Models", Challenge 1 (select the rows
  routed to an expert, run the expert MLP, weight by the routing
  probability, index-add into token order), without and with MXFP8 round
  trips on the operands.
* P3: identity-weight expert with probability 1 reduces to silu(gate)*up.
* P4: invariants -- split_sizes sum to T*k, the permutation is a
  bijection, quantise-then-permute equals permute-then-quantise, expert
  relabelling does not change the output.
* P5: backward against central finite differences of the unquantised
  forward, and d(prob) against its closed form <dY_t, y_r> / p_r.
* P6: edge cases (empty experts, one-row groups, all tokens on one
  expert, K = 2880 tails).
"""
import numpy as np
import pytest

from mxfp8_grouped_gemm_x32_b200.workloads import (bf16_bits_to_f32, get_config,
                                                   make_inputs)
from oracle import moe, mxfp8


def _vals(inp):
    f = lambda k: bf16_bits_to_f32(inp[k]).astype(np.float64)
    return f("x"), f("w1"), f("w2"), f("dy")


def _hf_loop(x, w1, w2, idx, prob, qx=None, qw=None, qh=None):
    """The Hugging Face per-expert loop, restated in float64.  The routing
    weight is applied inside the activation (ScaledSwiGLU) -- the same
    product as weighting the expert output, since the down projection is
    linear.  q* are optional MXFP8 round trips for x, weights and h."""
    qx = qx or (lambda v: v)
    qw = qw or (lambda v: v)
    qh = qh or (lambda v: v)
    T, H = x.shape
    E = w1.shape[0]
    I = w1.shape[1] // 2
    final = np.zeros((T, w2.shape[1]))
    expert_mask = np.zeros((E, idx.shape[1], T), bool)          # one-hot
    for t in range(T):
        for j in range(idx.shape[1]):
            expert_mask[idx[t, j], j, t] = True
    for e in range(E):
        which, top_x = np.where(expert_mask[e])                   # (choice, token)
        if top_x.size == 0:
            continue
        order = np.lexsort((which, top_x))                       # token-major
        which, top_x = which[order], top_x[order]
        cur = qx(x[top_x])
        gate = cur @ qw(w1[e, :I]).T
        up = cur @ qw(w1[e, I:]).T
        act = prob[top_x, which][:, None] * (gate / (1 + np.exp(-gate))) * up
        hidden = qh(act) @ qw(w2[e]).T
        np.add.at(final, top_x, hidden)
    return final


@pytest.fixture(scope="module")
def tiny():
    cfg = get_config("tiny")
    inp = make_inputs(cfg, seed=0)
    return cfg, inp


def test_forward_equals_hf_loop_unquantised(tiny):
    cfg, inp = tiny
    x, w1, w2, _ = _vals(inp)
    ref = _hf_loop(x, w1, w2, inp["topk_idx"], inp["topk_prob"].astype(np.float64))
    got = moe.forward(x, w1, w2, inp["topk_idx"], inp["topk_prob"], quantize=False)["out"]
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_forward_equals_hf_loop_on_roundtripped_operands(tiny):
    cfg, inp = tiny
    x, w1, w2, _ = _vals(inp)
    q = mxfp8.roundtrip_rows
    ref = _hf_loop(x, w1, w2, inp["topk_idx"], inp["topk_prob"].astype(np.float64),
                   qx=q, qw=q, qh=q)
    got = moe.forward(x, w1, w2, inp["topk_idx"], inp["topk_prob"])["out"]
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_quantised_forward_close_to_unquantised(tiny):
    cfg, inp = tiny
    x, w1, w2, _ = _vals(inp)
    a = moe.forward(x, w1, w2, inp["topk_idx"], inp["topk_prob"])["out"]
    b = moe.forward(x, w1, w2, inp["topk_idx"], inp["topk_prob"], quantize=False)["out"]
    rel = np.sqrt(np.mean((a - b) ** 2)) / np.sqrt(np.mean(b ** 2))
    assert 1e-3 < rel < 0.1          # MXFP8 noise: present, but small


def test_identity_expert_closed_form():
    """H = 2I, W1 = identity, W2 = [I_I; 0], p = 1: y = [silu(x1) x2; 0]
    with x MX-exact (E4M3 codes times a power of two) so x's round trip is
    the identity; the output is then exactly the round trip of the closed
    form silu(x1) * x2 padded with zeros."""
    I, H, T = 64, 128, 8
    rng = np.random.default_rng(7)
    codes = rng.integers(0x20, 0x50, (T, H)).astype(np.uint8) | (rng.integers(0, 2, (T, H)).astype(np.uint8) << 7)
    codes[:, ::32] = 0x7E
    x = mxfp8.e4m3_decode(codes) * 2.0 ** -6
    w1 = np.eye(2 * I)[None]
    w2 = np.concatenate([np.eye(I), np.zeros((H - I, I))], axis=0)[None]
    idx = np.zeros((T, 1), np.int32)
    prob = np.ones((T, 1), np.float32)
    out = moe.forward(x, w1, w2, idx, prob)["out"]
    h = x[:, :I] / (1 + np.exp(-x[:, :I])) * x[:, I:]
    want = np.concatenate([mxfp8.roundtrip_rows(h), np.zeros((T, H - I))], axis=1)
    assert np.array_equal(out, want)


def test_identity_expert_bf16_path():
    """BF16 recipe (no MXFP8, h kept in bf16): with the identity expert the
    output is h = silu(x1) x2 rounded to bf16, checked against the
    definition of round-to-nearest-even by brute force over the neighbouring
    bf16 values, not against the oracle's own rounding."""
    I, H, T = 64, 128, 16
    rng = np.random.default_rng(8)
    x = rng.standard_normal((T, H))
    w1 = np.eye(2 * I)[None]
    w2 = np.concatenate([np.eye(I), np.zeros((H - I, I))], axis=0)[None]
    idx = np.zeros((T, 1), np.int32)
    prob = np.ones((T, 1), np.float32)
    out = moe.forward(x, w1, w2, idx, prob, quantize=False, h_bf16=True)["out"]
    h = x[:, :I] / (1 + np.exp(-x[:, :I])) * x[:, I:]
    assert np.all(out[:, I:] == 0)
    v = out[:, :I]
    bits = v.astype(np.float32).view(np.uint32)
    assert np.all(v.astype(np.float32).astype(np.float64) == v) and np.all(bits & 0xFFFF == 0)   # bf16 values
    nb = bits >> 16
    for step in (-1, 1):                        # neighbours one bf16 step down and up
        w = ((nb.astype(np.int64) + step).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        dv, dw = np.abs(v - h), np.abs(w - h)
        assert np.all((dv < dw) | ((dv == dw) & (nb % 2 == 0)))
    # without the bf16 step h passes through unrounded
    out2 = moe.forward(x, w1, w2, idx, prob, quantize=False)["out"]
    assert np.allclose(out2[:, :I], h, rtol=1e-15, atol=0)


def _is_rne_bf16_of(v, exact):
    """v holds the bf16 values nearest to `exact` (ties to even), checked by
    brute force over the neighbouring bf16 values."""
    bits = v.astype(np.float32).view(np.uint32)
    if not (np.all(v.astype(np.float32).astype(np.float64) == v) and np.all(bits & 0xFFFF == 0)):
        return False
    nb = bits >> 16
    for step in (-1, 1):
        w = ((nb.astype(np.int64) + step).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        dv, dw = np.abs(v - exact), np.abs(w - exact)
        if not np.all((dv < dw) | ((dv == dw) & (nb % 2 == 0))):
            return False
    return True


def test_identity_expert_bf16_backward():
    """BF16 recipe backward (da and the recomputed h held in bf16): with the
    identity expert (W_gate_up = I, W_down = [I; 0], p = 1, k = 1) dX is
    da = [dg, du] rounded to bf16 and dW_down's top block is dy1^T bf16(h),
    with dg, du, h written out here from the ScaledSwiGLU backward's
    definition (the saved activation A = x in bf16)."""
    I, T = 32, 24
    H = 2 * I
    rng = np.random.default_rng(9)
    x = moe.bf16_round(rng.standard_normal((T, H)))
    dy = moe.bf16_round(rng.standard_normal((T, H)))
    w1 = np.eye(2 * I)[None]
    w2 = np.concatenate([np.eye(I), np.zeros((H - I, I))], axis=0)[None]
    idx = np.zeros((T, 1), np.int32)
    prob = np.ones((T, 1), np.float32)
    fwd = moe.forward(x, w1, w2, idx, prob, quantize=False, h_bf16=True)
    b = moe.backward(fwd, x, w1, w2, prob, dy, quantize=False, bf16_held=True)
    g, u, dh = x[:, :I], x[:, I:], dy[:, :I]
    sig = 1.0 / (1.0 + np.exp(-g))
    dg = dh * u * sig * (1.0 + g * (1.0 - sig))
    du = dh * g * sig
    h = g * sig * u
    assert _is_rne_bf16_of(b["dX"][:, :I], dg) and _is_rne_bf16_of(b["dX"][:, I:], du)
    assert _is_rne_bf16_of(b["h_b"], h)
    assert np.allclose(b["dW2"][0][:I], dy[:, :I].T @ b["h_b"], rtol=1e-12, atol=0)
    assert np.all(b["dW2"][0][I:] == dy[:, I:].T @ b["h_b"])
    # without the bf16 step da passes through unrounded
    b2 = moe.backward(fwd, x, w1, w2, prob, dy, quantize=False)
    assert np.allclose(b2["dX"][:, :I], dg, rtol=1e-13, atol=0)


def test_bf16_backward_scales_exactly_with_dy():
    """BF16 recipe backward: dY -> 2^5 dY multiplies every gradient by exactly
    2^5 (bf16 rounding commutes with a power-of-two scale; h does not depend
    on dY) -- a dropped or doubled term of the dY path breaks this."""
    x, w1, w2, idx, prob, _ = _small_layer(seed=21)
    rng = np.random.default_rng(22)
    dy = moe.bf16_round(rng.standard_normal(x.shape))
    fwd = moe.forward(x, w1, w2, idx, prob, quantize=False, h_bf16=True)
    a = moe.backward(fwd, x, w1, w2, prob, dy, quantize=False, bf16_held=True)
    b = moe.backward(fwd, x, w1, w2, prob, 32.0 * dy, quantize=False, bf16_held=True)
    for key in ("dX", "dW1", "dW2", "dprob_f64", "da"):
        assert np.array_equal(b[key], 32.0 * a[key]), key
    assert np.array_equal(b["h_b"], a["h_b"])


def test_bf16_backward_close_to_the_exact_gradient():
    """The bf16 roundings of da and h change each gradient by at most a few
    bf16 steps: within 2 % of the rms of the unrounded backward, element by
    element (an index or sign mistake in the rounded path gives errors of the
    order of the rms)."""
    x, w1, w2, idx, prob, _ = _small_layer(seed=23, T=40)
    rng = np.random.default_rng(24)
    dy = moe.bf16_round(rng.standard_normal(x.shape))
    fwd = moe.forward(x, w1, w2, idx, prob, quantize=False, h_bf16=True)
    held = moe.backward(fwd, x, w1, w2, prob, dy, quantize=False, bf16_held=True)
    exact = moe.backward(fwd, x, w1, w2, prob, dy, quantize=False)
    for key in ("dX", "dW1", "dW2"):
        rms = np.sqrt(np.mean(exact[key] ** 2))
        assert np.max(np.abs(held[key] - exact[key])) <= 2e-2 * rms, key
    assert np.array_equal(held["dprob_f64"], exact["dprob_f64"])       # dprob does not use da or h


def test_permutation_invariants(tiny):
    cfg, inp = tiny
    perm, split = moe.permute(inp["topk_idx"], cfg.E)
    assert split.sum() == cfg.T * cfg.k
    assert np.array_equal(np.sort(perm), np.arange(cfg.T * cfg.k))
    flat = inp["topk_idx"].reshape(-1)
    offs = moe.offsets(split)
    for e in range(cfg.E):
        rows = perm[offs[e]:offs[e + 1]]
        assert np.all(flat[rows] == e) and np.all(np.diff(rows) > 0)   # stable


def test_quantise_commutes_with_permutation(tiny):
    cfg, inp = tiny
    x, w1, w2, _ = _vals(inp)
    f = moe.forward(x, w1, w2, inp["topk_idx"], inp["topk_prob"])
    c, s = mxfp8.quantize_rows(x)
    assert np.array_equal(f["xq_codes"], c[f["tok"]])
    assert np.array_equal(f["xq_scales"], s[f["tok"]])


def test_expert_relabelling_invariance(tiny):
    cfg, inp = tiny
    x, w1, w2, _ = _vals(inp)
    pi = np.array([2, 0, 3, 1])
    out = moe.forward(x, w1, w2, inp["topk_idx"], inp["topk_prob"])["out"]
    w1p, w2p = np.empty_like(w1), np.empty_like(w2)
    w1p[pi], w2p[pi] = w1, w2
    out2 = moe.forward(x, w1p, w2p, pi[inp["topk_idx"]].astype(np.int32), inp["topk_prob"])["out"]
    assert np.allclose(out, out2, rtol=0, atol=1e-12 * np.abs(out).max())


def _small_layer(seed=11, T=6, H=64, I=32, E=3, k=2):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H))
    w1 = rng.standard_normal((E, 2 * I, H)) / np.sqrt(H)
    w2 = rng.standard_normal((E, H, I)) / np.sqrt(I)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    prob = rng.uniform(0.2, 0.8, (T, k))
    dy = rng.standard_normal((T, H))
    return x, w1, w2, idx, prob, dy


def test_backward_matches_finite_differences():
    x, w1, w2, idx, prob, dy = _small_layer()

    def loss(x_, w1_, w2_, p_):
        f = moe.forward(x_, w1_, w2_, idx, p_, quantize=False, round_saved=False)
        return np.sum(f["out"] * dy)

    f = moe.forward(x, w1, w2, idx, prob, quantize=False, round_saved=False)
    g = moe.backward(f, x, w1, w2, prob, dy, quantize=False)
    rng = np.random.default_rng(12)
    eps = 1e-6

    def check(arr, grad, name, n=12):
        for _ in range(n):
            i = tuple(rng.integers(0, s) for s in arr.shape)
            old = arr[i]
            arr[i] = old + eps
            lp = loss(x, w1, w2, prob)
            arr[i] = old - eps
            lm = loss(x, w1, w2, prob)
            arr[i] = old
            num = (lp - lm) / (2 * eps)
            assert abs(num - grad[i]) <= 1e-6 * max(1.0, abs(num)), (name, i, num, grad[i])

    check(x, g["dX"], "dX")
    check(w1, g["dW1"], "dW1")
    check(w2, g["dW2"], "dW2")
    check(prob, g["dprob_f64"], "dprob")


def test_dprob_closed_form():
    """d(prob) of slot (t, j) = <dY_t, y_r> / p_r, y_r the weighted expert row."""
    x, w1, w2, idx, prob, dy = _small_layer(seed=13)
    f = moe.forward(x, w1, w2, idx, prob, quantize=False, round_saved=False)
    g = moe.backward(f, x, w1, w2, prob, dy, quantize=False)
    k = idx.shape[1]
    for r, slot in enumerate(f["perm"]):
        t, j = divmod(slot, k)
        want = np.dot(dy[t], f["Y"][r]) / prob[t, j]
        assert abs(g["dprob_f64"][t, j] - want) <= 1e-10 * max(1, abs(want))


def test_quantised_backward_close_to_unquantised(tiny):
    cfg, inp = tiny
    x, w1, w2, dy = _vals(inp)
    fq = moe.forward(x, w1, w2, inp["topk_idx"], inp["topk_prob"])
    gq = moe.backward(fq, x, w1, w2, inp["topk_prob"], dy)
    fe = moe.forward(x, w1, w2, inp["topk_idx"], inp["topk_prob"], quantize=False, round_saved=False)
    ge = moe.backward(fe, x, w1, w2, inp["topk_prob"], dy, quantize=False)
    for key in ("dX", "dW1", "dW2", "dprob_f64"):
        a, b = gq[key], ge[key]
        rel = np.sqrt(np.mean((a - b) ** 2)) / np.sqrt(np.mean(b ** 2))
        assert rel < 0.15, (key, rel)


def test_edge_cases_empty_single_all_on_one():
    """Expert 1 empty, expert 2 receives exactly one row, everything else
    on expert 0; the per-expert results equal a dense computation of that
    expert alone and the empty expert's weight gradients are zero."""
    cfg = get_config("tiny", T=64, H=64, I=64, E=3, k=1)
    idx = np.zeros((64, 1), np.int32)
    idx[5, 0] = 2
    inp = make_inputs(cfg, seed=3, topk_idx=idx)
    x, w1, w2, dy = _vals(inp)
    f = moe.forward(x, w1, w2, inp["topk_idx"], inp["topk_prob"])
    assert list(f["split_sizes"]) == [63, 0, 1]
    g = moe.backward(f, x, w1, w2, inp["topk_prob"], dy)
    assert np.all(g["dW1"][1] == 0) and np.all(g["dW2"][1] == 0)
    # the single row of expert 2 is token 5
    r = f["offsets"][2]
    assert f["tok"][r] == 5
    xd = mxfp8.roundtrip_rows(x[5:6])
    a = xd @ mxfp8.roundtrip_rows(w1[2]).T
    assert np.array_equal(f["A"][r:r + 1], a)


def test_k2880_tail_shapes():
    """K = 2880 = 90 blocks of 32 (not a multiple of 128) in both GEMMs."""
    cfg = get_config("gpt_oss_20b", T=16, E=4, k=2)
    inp = make_inputs(cfg, seed=1)
    x, w1, w2, dy = _vals(inp)
    f = moe.forward(x, w1, w2, inp["topk_idx"], inp["topk_prob"], experts=[0, 1])
    assert f["xq_scales"].shape == (32, 90) and f["hq_scales"].shape == (32, 90)
    ref = _hf_loop(x, w1[:2], w2[:2], np.where(inp["topk_idx"] < 2, inp["topk_idx"], 0),
                   np.where(inp["topk_idx"] < 2, inp["topk_prob"], 0).astype(np.float64),
                   qx=mxfp8.roundtrip_rows, qw=mxfp8.roundtrip_rows, qh=mxfp8.roundtrip_rows)
    assert np.max(np.abs(f["out"] - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_bf16_rounding_single_step():
    """float64 -> bf16 rounds once (no double rounding through float32)."""
    v = np.array([1.0 + 2 ** -8 + 2 ** -30, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0, 3.0e38 * 1.2])
    got = moe.bf16_value(moe.bf16_bits(v))
    assert got[0] == 1.0 + 2 ** -7          # above the tie -> up
    assert got[1] == 1.0                    # tie -> even
    assert got[2] == 1.0 + 4 * 2 ** -8      # tie -> even (up)
    assert got[3] == -2.5 and got[4] == 0.0 and np.isinf(got[5])
