"""The BF16 recipe's grouped forward (moe_grouped_mlp_fwd_bf16: bf16 operands,
no MXFP8, h kept in bf16) against the oracle in the same mode, through the C
ABI.  Bars: max|gpu - oracle| / rms(oracle) <= 2e-2 and
rms(gpu - oracle) / rms(oracle) <= 1e-2 (the output bar of the MXFP8 path;
the remaining differences are fp32 accumulation order and the bf16 rounding
of h and of out)."""
import numpy as np
import pytest

from mxfp8_grouped_gemm_x32_b200.workloads import bf16_bits_to_f32, get_config, make_inputs
from oracle import moe as omoe

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": dict(),
    "gptoss_k2880": dict(name="gpt_oss_20b", T=160, E=4, k=2),
    "ragged_128e": dict(name="qwen3_30b_ragged", T=96, H=256, I=256, E=128, k=8),
}


@pytest.mark.parametrize("case", list(CASES))
def test_bf16_forward_matches_oracle(case):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mxfp8_grouped_gemm_x32_b200 import lib
    from mxfp8_grouped_gemm_x32_b200.layer import GroupedMLP
    over = dict(CASES[case])
    cfg = get_config(over.pop("name", "tiny"), **over)
    inp = make_inputs(cfg, seed=21)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    L = GroupedMLP(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, backward=False, guard=4096)
    L.permute_index(torch.from_numpy(inp["topk_idx"]).cuda(), torch.from_numpy(inp["topk_prob"]).cuda())
    out = L.forward_bf16(bf(inp["x"]), bf(inp["w1"]), bf(inp["w2"]))
    torch.cuda.synchronize()
    assert lib.moe_get_device_status(0) == 0
    assert L.check_guards() == []
    f64 = lambda k: bf16_bits_to_f32(inp[k]).astype(np.float64)
    ref = omoe.forward(f64("x"), f64("w1"), f64("w2"), inp["topk_idx"], inp["topk_prob"], quantize=False,
                       h_bf16=True)["out"]
    g = out.float().cpu().numpy().astype(np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(g - ref)) / rms <= 2e-2
    assert np.sqrt(np.mean((g - ref) ** 2)) / rms <= 1e-2
