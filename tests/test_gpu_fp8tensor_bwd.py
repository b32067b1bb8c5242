"""The per-tensor FP8 recipe's backward (moe_grouped_mlp_bwd_fp8_tensor),
after its forward saved A, against the oracle of the same recipe
(oracle/fp8tensor.py: backward), through the C ABI.

Bars: dY's factor bit-exact; the factors of da and h within one bf16 step of
the oracle's (their |max| is taken from fp32 values on the GPU and float64
ones in the oracle before the bf16 rounding) and, on these seeds, equal;
dX, dW1, dW2, dprob: max|gpu - oracle| / rms(oracle) <= 2e-2 after the
element-wise allowance of `ambiguity.backward_allowance_f8t` (bf16 values of
A, da and h that lie within the kernels' fp32 error band of a rounding
boundary, propagated through the per-tensor round trip and the next GEMM;
from oracle values only) and rms(gpu - oracle) / rms(oracle) <= 1e-2 with
none; the weight gradients of experts without tokens exactly zero."""
import numpy as np
import pytest

from mxfp8_grouped_gemm_x32_b200.workloads import bf16_bits_to_f32, get_config, make_inputs
from oracle import fp8tensor as ft

from . import ambiguity

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": dict(),
    "gptoss_k2880": dict(name="gpt_oss_20b", T=160, E=4, k=2),
    "ragged_128e": dict(name="qwen3_30b_ragged", T=96, H=256, I=256, E=128, k=8),
    "one_token": dict(T=1),
}

_RUNS = {}


def _run(case):
    if case in _RUNS:
        return _RUNS[case]
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mxfp8_grouped_gemm_x32_b200 import lib
    from mxfp8_grouped_gemm_x32_b200.layer import GroupedMLP
    over = dict(CASES[case])
    cfg = get_config(over.pop("name", "tiny"), **over)
    inp = make_inputs(cfg, seed=29)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    L = GroupedMLP(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, backward=True, guard=4096)
    x, w1, w2, dy = bf(inp["x"]), bf(inp["w1"]), bf(inp["w2"]), bf(inp["dy"])
    L.permute_index(torch.from_numpy(inp["topk_idx"]).cuda(), torch.from_numpy(inp["topk_prob"]).cuda())
    L.forward_fp8_tensor(x, w1, w2)
    dX, dW1, dW2, dprob = L.backward_fp8_tensor(dy, x, w1, w2)
    torch.cuda.synchronize()
    assert lib.moe_get_device_status(0) == 0
    assert L.check_guards() == []
    f64 = lambda k: bf16_bits_to_f32(inp[k]).astype(np.float64)
    f = ft.forward(f64("x"), f64("w1"), f64("w2"), inp["topk_idx"], inp["topk_prob"])
    b = ft.backward(f, f64("dy"), inp["topk_prob"])
    g = lambda t: t.float().cpu().numpy().astype(np.float64)
    res = dict(cfg=cfg, inp=inp, f=f, b=b, dX=g(dX), dW1=g(dW1), dW2=g(dW2), dprob=g(dprob),
               sc=L.fp8_bwd_scales.cpu().numpy(), split=L.split_sizes.cpu().numpy())
    res["allow"] = ambiguity.backward_allowance_f8t(f, b, f64("dy"), inp["topk_idx"])
    _RUNS[case] = res
    return res


@pytest.mark.parametrize("case", list(CASES))
def test_backward_factors(case):
    r = _run(case)
    sc, b = r["sc"], r["b"]
    assert sc[0] == b["s_dy"]
    for got, want in ((sc[1], b["s_da"]), (sc[2], b["s_hb"])):
        assert abs(float(got) / float(want) - 1.0) <= 2.0 ** -7
        assert got == want


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("key,ref", [("dX", "dX"), ("dW1", "dW1"), ("dW2", "dW2"), ("dprob", "dprob_f64")])
def test_fp8_tensor_backward_matches_oracle(case, key, ref):
    r = _run(case)
    mx = ambiguity.within(r[key], r["b"][ref], 2e-2, r["allow"][key], bf16_out=key != "dprob")
    assert mx <= 2e-2, mx
    want = r["b"][ref]
    rr = np.sqrt(np.mean((r[key] - want) ** 2)) / np.sqrt(np.mean(want ** 2))
    assert rr <= 1e-2, rr


@pytest.mark.parametrize("case", list(CASES))
def test_empty_experts_have_zero_weight_gradients(case):
    r = _run(case)
    empty = np.flatnonzero(r["split"] == 0)
    assert np.all(r["dW1"][empty] == 0.0) and np.all(r["dW2"][empty] == 0.0)


@pytest.mark.parametrize("recipe", ["bf16", "fp8_tensor"])
def test_zero_tokens(recipe):
    """A batch with no tokens runs every launch of both recipes' forward and
    backward and leaves zero weight gradients."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mxfp8_grouped_gemm_x32_b200 import lib
    from mxfp8_grouped_gemm_x32_b200.layer import GroupedMLP
    cfg = get_config("tiny", T=0)
    inp = make_inputs(cfg, seed=31)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    L = GroupedMLP(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, backward=True, guard=4096)
    x, w1, w2, dy = bf(inp["x"]), bf(inp["w1"]), bf(inp["w2"]), bf(inp["dy"])
    L.permute_index(torch.from_numpy(inp["topk_idx"]).cuda(), torch.from_numpy(inp["topk_prob"]).cuda())
    getattr(L, "forward_" + recipe)(x, w1, w2)
    dX, dW1, dW2, dprob = getattr(L, "backward_" + recipe)(dy, x, w1, w2)
    torch.cuda.synchronize()
    assert lib.moe_get_device_status(0) == 0
    assert L.check_guards() == []
    assert dX.shape == (0, cfg.H) and dprob.shape == (0, cfg.k)
    assert float(dW1.float().abs().max()) == 0.0 and float(dW2.float().abs().max()) == 0.0
