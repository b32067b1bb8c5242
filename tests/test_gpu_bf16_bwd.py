"""The BF16 recipe's backward (moe_grouped_mlp_bwd_bf16: bf16 operands, no
MXFP8; da = [dg, du] and the recomputed h held in bf16) against the oracle in
the same mode (backward with quantize=False, bf16_held=True), through the C
ABI, after the BF16 forward that saves A.

Bars: the saved A is the bf16 rounding of A (an fp32 accumulation next to the
oracle's exact value: a rounding decision may go the other way, so each
element is within one bf16 step of the oracle's, plus 1e-4 rms for the
accumulation error of near-zero elements, and at most 1 % differ);
dX, dW1, dW2, dprob: max|gpu - oracle| / rms(oracle) <= 2e-2 after an
element-wise allowance and rms(gpu - oracle) / rms(oracle) <= 1e-2 with
none.  The allowance (tests/ambiguity.py, from oracle values only) holds the
output's own bf16 rounding and, propagated through the GEMM that follows,
each bf16 value of the saved A, da and h whose float64 value lies within the
kernels' fp32 error band of a rounding boundary (it may round either way);
what remains is fp32 accumulation order.  The weight gradients of experts
without tokens are exactly zero."""
import numpy as np
import pytest

from mxfp8_grouped_gemm_x32_b200.workloads import bf16_bits_to_f32, get_config, make_inputs
from oracle import moe as omoe

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
    inp = make_inputs(cfg, seed=23)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    L = GroupedMLP(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, backward=True, guard=4096)
    x, w1, w2, dy = bf(inp["x"]), bf(inp["w1"]), bf(inp["w2"]), bf(inp["dy"])
    L.permute_index(torch.from_numpy(inp["topk_idx"]).cuda(), torch.from_numpy(inp["topk_prob"]).cuda())
    L.forward_bf16(x, w1, w2)
    dX, dW1, dW2, dprob = L.backward_bf16(dy, x, w1, w2)
    torch.cuda.synchronize()
    assert lib.moe_get_device_status(0) == 0
    assert L.check_guards() == []
    f64 = lambda k: bf16_bits_to_f32(inp[k]).astype(np.float64)
    f = omoe.forward(f64("x"), f64("w1"), f64("w2"), inp["topk_idx"], inp["topk_prob"], quantize=False,
                     h_bf16=True)
    b = omoe.backward(f, f64("x"), f64("w1"), f64("w2"), inp["topk_prob"], f64("dy"), quantize=False,
                      bf16_held=True)
    def g(t):
        with np.errstate(invalid="ignore"):   # padding rows of the saved A are never written (any bits)
            return t.float().cpu().numpy().astype(np.float64)

    res = dict(cfg=cfg, inp=inp, f=f, b=b, dX=g(dX), dW1=g(dW1), dW2=g(dW2), dprob=g(dprob),
               saved=g(L.saved_a[: int(L.group_offsets[cfg.E])]), go=L.group_offsets.cpu().numpy(),
               split=L.split_sizes.cpu().numpy())
    _RUNS[case] = res
    return res


def _rel_rms(g, ref):
    return np.sqrt(np.mean((g - ref) ** 2)) / np.sqrt(np.mean(ref ** 2))


@pytest.mark.parametrize("case", list(CASES))
def test_saved_a_is_bf16_of_a(case):
    r = _run(case)
    f, go, split = r["f"], r["go"], r["split"]
    E = r["cfg"].E
    perm_rows = np.concatenate([np.arange(go[e], go[e] + split[e]) for e in range(E)])
    got = r["saved"][perm_rows]
    ref = f["saved"]                                   # bf16 of the exact A, permuted order
    # one bf16 step (at most) around the value, plus the fp32 accumulation
    # error of a near-zero element (K <= 2880 products, each <= 1e-1 here)
    step = np.abs(ref) * 2.0 ** -7 + 1e-4 * np.sqrt(np.mean(ref ** 2))
    assert np.all(np.abs(got - ref) <= step)
    assert np.mean(got != ref) <= 1e-2


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("key,ref", [("dX", "dX"), ("dW1", "dW1"), ("dW2", "dW2"), ("dprob", "dprob_f64")])
def test_bf16_backward_matches_oracle(case, key, ref):
    r = _run(case)
    if "allow" not in r:
        f64 = lambda k: bf16_bits_to_f32(r["inp"][k]).astype(np.float64)
        r["allow"] = ambiguity.backward_allowance_bf16(r["f"], r["b"], f64("x"), f64("w1"), f64("w2"), f64("dy"),
                                                       r["inp"]["topk_idx"])
    mx = ambiguity.within(r[key], r["b"][ref], 2e-2, r["allow"][key], bf16_out=key != "dprob")
    assert mx <= 2e-2, mx
    rr = _rel_rms(r[key], r["b"][ref])
    assert rr <= 1e-2, rr


@pytest.mark.parametrize("case", list(CASES))
def test_empty_experts_have_zero_weight_gradients(case):
    r = _run(case)
    empty = np.flatnonzero(r["split"] == 0)
    assert np.all(r["dW1"][empty] == 0.0) and np.all(r["dW2"][empty] == 0.0)
