"""The seeded input recipe shared by the oracle's and the CUDA path's tests
(mxfp8_grouped_gemm_x32_b200/workloads.py): deterministic, independent of the
thread count, bf16-rounded with round-to-nearest-even, and drawn with the
stated distributions and routing."""
import numpy as np

from mxfp8_grouped_gemm_x32_b200 import workloads as wl


def test_deterministic_and_seed_dependent():
    cfg = wl.get_config("tiny")
    a, b = wl.make_inputs(cfg, seed=5), wl.make_inputs(cfg, seed=5)
    for key in a:
        assert np.array_equal(a[key], b[key]), key
    c = wl.make_inputs(cfg, seed=6)
    assert not np.array_equal(a["x"], c["x"])


def test_chunked_draws_do_not_depend_on_the_thread_count(monkeypatch):
    n = 3 * wl._CHUNK + 123                      # several chunks and a ragged last one
    many = wl._normal_f32(1, 2, n, 0.5)
    monkeypatch.setattr(wl.os, "sched_getaffinity", lambda pid: {0})
    one = wl._normal_f32(1, 2, n, 0.5)
    assert np.array_equal(many, one)


def test_bf16_rounding_is_nearest_even():
    f = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, np.inf, np.nan], np.float32)
    bits = wl.bf16_bits_from_f32(f)
    back = wl.bf16_bits_to_f32(bits)
    assert back[0] == 1.0
    assert back[1] == 1.0                        # tie -> even mantissa
    assert back[2] == 1.0 + 2.0 ** -6            # tie -> even mantissa (upwards)
    assert back[3] == -2.5 and np.isinf(back[4]) and np.isnan(back[5])


def test_distributions_and_routing():
    cfg = wl.get_config("tiny", T=2048)
    inp = wl.make_inputs(cfg, seed=0)
    x = wl.bf16_bits_to_f32(inp["x"]).astype(np.float64)
    w1 = wl.bf16_bits_to_f32(inp["w1"]).astype(np.float64)
    w2 = wl.bf16_bits_to_f32(inp["w2"]).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    assert abs(w1.std() * np.sqrt(cfg.H) - 1.0) < 0.02              # N(0, 1/fan_in)
    assert abs(w2.std() * np.sqrt(cfg.I) - 1.0) < 0.02
    idx, prob = inp["topk_idx"], inp["topk_prob"]
    assert idx.shape == (cfg.T, cfg.k) and idx.dtype == np.int32 and prob.dtype == np.float32
    assert np.all((idx >= 0) & (idx < cfg.E))
    assert np.all(idx[:, 0] != idx[:, 1])                           # k distinct experts per token
    assert np.allclose(prob.sum(axis=1), 1.0, atol=1e-6)            # renormalised
    assert np.all(prob[:, 0] >= prob[:, 1])                         # descending
    # the routing is the top-k of the stored logits
    lg = inp["router_logits"].astype(np.float64)
    top = np.argsort(-lg, axis=1, kind="stable")[:, :cfg.k]
    assert np.array_equal(top, idx)


def test_skewed_router_empties_experts():
    cfg = wl.get_config("qwen3_profile")
    inp = wl.make_inputs(cfg, seed=0, weights=False, grad=False)
    counts = np.bincount(inp["topk_idx"].ravel(), minlength=cfg.E)
    assert counts.sum() == cfg.T * cfg.k
    # the per-expert bias (std 1.5) leaves experts empty and gives a long tail of large groups
    assert (counts == 0).sum() >= 10
    assert counts.max() > 50 * np.median(counts)
