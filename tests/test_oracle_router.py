"""Pins of the oracle's router (oracle/router.py) against things other than
itself: brute force over every k-subset of experts on tiny rows, the closed
form (a softmax over the kept logits), torch.topk + torch.softmax on random
rows, exact ties, invariants (shift, relabelling), and rows with -inf / NaN.
"""
import itertools

import numpy as np
import pytest

from oracle import router


def _brute(row, k):
    """The k-subset with the largest total softmax probability, listed in
    descending probability, ties to the lower id -- by enumeration."""
    E = row.size
    key = np.where(np.isnan(row), -np.inf, row)
    m = np.max(key)
    p = np.exp(key - (m if np.isfinite(m) else 0.0))
    p = p / p.sum()
    best = None
    for sub in itertools.combinations(range(E), k):
        # lexicographic preference: larger probabilities first, then lower ids
        srt = sorted(sub, key=lambda e: (-key[e], e))
        score = tuple(-key[e] for e in srt) + tuple(srt)
        if best is None or score < best[0]:
            best = (score, srt)
    sel = np.array(best[1])
    return sel, p[sel] / p[sel].sum()


def test_brute_force_tiny():
    rng = np.random.default_rng(0)
    for E in (2, 3, 5, 8):
        for k in range(1, min(E, 4) + 1):
            lg = rng.normal(size=(20, E))
            lg[::3, 0] = lg[::3, 1]          # exact ties
            lg[1::4, :] = np.round(lg[1::4, :])  # many ties
            idx, prob = router.route_topk(lg, k)
            for t in range(lg.shape[0]):
                sel, p = _brute(lg[t], k)
                assert np.array_equal(idx[t], sel), (E, k, t)
                assert np.allclose(prob[t], p, rtol=1e-13, atol=0)


def test_closed_form_softmax_of_kept_logits():
    rng = np.random.default_rng(1)
    lg = rng.normal(size=(64, 128)) * 3 + rng.normal(size=128) * 1.5
    idx, prob = router.route_topk(lg, 8)
    kept = np.take_along_axis(lg, idx, axis=1)
    z = np.exp(kept - kept.max(axis=1, keepdims=True))
    assert np.allclose(prob, z / z.sum(axis=1, keepdims=True), rtol=1e-13, atol=0)
    assert np.allclose(prob.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    assert np.all(np.diff(prob, axis=1) <= 0)
    assert all(len(set(r)) == 8 for r in idx)


def test_against_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(2)
    lg = rng.normal(size=(256, 32))
    idx, prob = router.route_topk(lg, 4)
    t = torch.from_numpy(lg)
    v, i = torch.topk(torch.softmax(t, dim=1), 4, dim=1)
    assert np.array_equal(idx, i.numpy())
    assert np.allclose(prob, (v / v.sum(dim=1, keepdim=True)).numpy(), rtol=1e-13, atol=0)


def test_invariants():
    rng = np.random.default_rng(3)
    lg = rng.normal(size=(50, 16))
    idx, prob = router.route_topk(lg, 3)
    i2, p2 = router.route_topk(lg + 7.25, 3)        # shift invariance
    assert np.array_equal(idx, i2) and np.allclose(prob, p2, rtol=1e-12, atol=0)
    perm = rng.permutation(16)                      # relabelling (distinct logits)
    i3, p3 = router.route_topk(lg[:, perm], 3)
    assert np.array_equal(perm[i3], idx) and np.allclose(p3, prob, rtol=1e-13, atol=0)
    i1, p1 = router.route_topk(lg, 1)               # k = 1: argmax, probability 1
    assert np.array_equal(i1[:, 0], np.argmax(lg, axis=1)) and np.all(p1 == 1.0)


def test_inf_and_nan_rank_last():
    lg = np.array([[0.0, -np.inf, 1.0, np.nan], [np.nan, np.nan, 2.0, -np.inf]])
    idx, prob = router.route_topk(lg, 2)
    assert idx.tolist() == [[2, 0], [2, 0]]
    e = np.exp(-1.0)
    assert np.allclose(prob[0], [1 / (1 + e), e / (1 + e)], rtol=1e-15)
    assert prob[1].tolist() == [1.0, 0.0]
