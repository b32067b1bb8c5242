"""The per-tensor FP8 recipe's grouped forward (moe_grouped_mlp_fwd_fp8_tensor)
against the oracle of the same recipe (oracle/fp8tensor.py), through the C
ABI.  Bars: the factors of x and of every expert's weights and the E4M3 codes
of x (permuted rows) and of the weights bit-exact; h's factor within one bf16
step of the oracle's (h is computed in fp32 on the GPU and in float64 in the
oracle before its bf16 rounding, so its |max| can differ by one bf16 step);
out: max|gpu - oracle| / rms(oracle) <= 2e-2 and rms(gpu - oracle) / rms <=
1e-2, the output bar of the MXFP8 path."""
import numpy as np
import pytest

from mxfp8_grouped_gemm_x32_b200.workloads import bf16_bits_to_f32, get_config, make_inputs
from oracle import fp8tensor as ft

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": dict(),
    "gptoss_k2880": dict(name="gpt_oss_20b", T=160, E=4, k=2),
    "ragged_128e": dict(name="qwen3_30b_ragged", T=96, H=256, I=256, E=128, k=8),
}


def _align(n):
    return (n + 255) // 256 * 256


@pytest.mark.parametrize("case", list(CASES))
def test_fp8_tensor_forward_matches_oracle(case):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mxfp8_grouped_gemm_x32_b200 import lib
    from mxfp8_grouped_gemm_x32_b200.layer import GroupedMLP
    over = dict(CASES[case])
    cfg = get_config(over.pop("name", "tiny"), **over)
    inp = make_inputs(cfg, seed=23)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    L = GroupedMLP(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, backward=False, guard=4096)
    L.permute_index(torch.from_numpy(inp["topk_idx"]).cuda(), torch.from_numpy(inp["topk_prob"]).cuda())
    out = L.forward_fp8_tensor(bf(inp["x"]), bf(inp["w1"]), bf(inp["w2"]))
    torch.cuda.synchronize()
    assert lib.moe_get_device_status(0) == 0
    assert L.check_guards() == []
    f64 = lambda k: bf16_bits_to_f32(inp[k]).astype(np.float64)
    ref = ft.forward(f64("x"), f64("w1"), f64("w2"), inp["topk_idx"], inp["topk_prob"])
    E, H, I, rc = cfg.E, cfg.H, cfg.I, L.rows_cap
    sc = L.fp8_scales.cpu().numpy()
    assert sc[0] == ref["s_x"]
    assert np.array_equal(sc[2:2 + E], ref["s_w1"]) and np.array_equal(sc[2 + E:], ref["s_w2"])
    assert abs(float(sc[1]) / float(ref["s_h"]) - 1.0) <= 2.0 ** -7
    # codes in the workspace: x (permuted rows) first, then the weights
    ws = L.ws_f8t.cpu().numpy()
    go = L.group_offsets.cpu().numpy()
    r2s = L.row_to_slot.cpu().numpy()[: go[E]]
    xq = ws[: rc * H].reshape(rc, H)[: go[E]]
    routed = r2s >= 0
    assert np.array_equal(xq[routed], ref["xq"][r2s[routed] // cfg.k])
    assert np.all(xq[~routed] == 0)
    o1 = _align(rc * H)
    assert np.array_equal(ws[o1:o1 + E * 2 * I * H].reshape(E, 2 * I, H), ref["w1q"])
    o2 = o1 + _align(E * 2 * I * H)
    assert np.array_equal(ws[o2:o2 + E * H * I].reshape(E, H, I), ref["w2q"])
    g = out.float().cpu().numpy().astype(np.float64)
    want = ref["out"]
    rms = np.sqrt(np.mean(want ** 2))
    assert np.max(np.abs(g - want)) / rms <= 2e-2
    assert np.sqrt(np.mean((g - want) ** 2)) / rms <= 1e-2
