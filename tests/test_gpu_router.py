"""Router (moe_router_topk) against the oracle's router on the same logits.

Bars: expert ids bit-exact (the selection compares input values only);
probabilities within 4e-6 relative.  That bound is derived from the fp32
arithmetic: the shift l_j - l_0 (one rounding), expf (<= 2 ulp), a sum of at
most 32 terms (<= 31 roundings) and a division -- (|l_j - l_0| + 35) * 2^-24
relative, under 4e-6 for logit spreads up to 30.
"""
import numpy as np
import pytest

from mxfp8_grouped_gemm_x32_b200.workloads import bf16_bits_from_f32, bf16_bits_to_f32, get_config, make_inputs
from oracle import router as orouter

pytestmark = pytest.mark.gpu
PROB_RTOL = 4e-6


def _run(logits_f32, k, bf16=False):
    import torch
    from mxfp8_grouped_gemm_x32_b200 import lib
    T, E = logits_f32.shape
    if bf16:
        bits = bf16_bits_from_f32(logits_f32)
        dev = torch.from_numpy(bits.view(np.int16)).cuda()
        ref_in = bf16_bits_to_f32(bits)
        dt = lib.MOE_DTYPE_BF16
    else:
        dev = torch.from_numpy(np.ascontiguousarray(logits_f32, dtype=np.float32)).cuda()
        ref_in = logits_f32
        dt = lib.MOE_DTYPE_F32
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    prob = torch.full((T, k), -7.0, dtype=torch.float32, device="cuda")
    lib.moe_router_topk(dev.data_ptr(), dt, T, E, k, idx.data_ptr(), prob.data_ptr(), 0)
    torch.cuda.synchronize()
    assert lib.moe_get_device_status(0) == 0
    ri, rp = orouter.route_topk(ref_in, k)
    return idx.cpu().numpy(), prob.cpu().numpy().astype(np.float64), ri, rp


def _check(gi, gp, ri, rp):
    assert np.array_equal(gi, ri)
    fin = np.isfinite(rp)
    assert np.array_equal(np.isfinite(gp), fin)
    assert np.all(np.abs(gp[fin] - rp[fin]) <= PROB_RTOL * np.abs(rp[fin]) + 1e-30)


@pytest.fixture(scope="module")
def cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("name", ["tiny", "gpt_oss_20b", "qwen3_30b_ragged", "mixtral_8x7b"])
def test_router_workload_logits(cuda, name):
    cfg = get_config(name)
    lg = make_inputs(cfg, seed=0, weights=False, grad=False)["router_logits"]
    _check(*_run(lg, cfg.k))


@pytest.mark.parametrize("E,k", [(256, 32), (256, 1), (8, 8), (33, 5), (1, 1), (200, 7)])
def test_router_shapes(cuda, E, k):
    rng = np.random.default_rng(E * 100 + k)
    lg = (rng.normal(size=(1000, E)) * 4).astype(np.float32)
    _check(*_run(lg, k))


def test_router_ties_inf_nan_bf16(cuda):
    rng = np.random.default_rng(5)
    lg = np.round(rng.normal(size=(2048, 64)) * 2).astype(np.float32) / 2   # many exact ties
    lg[::7, 3] = -np.inf
    lg[1::11, 5] = np.nan
    lg[2::13, :] = 1.0                                                      # all equal
    _check(*_run(lg, 6))
    _check(*_run(rng.normal(size=(777, 128)).astype(np.float32) * 3, 8, bf16=True))


def test_router_empty(cuda):
    import torch
    from mxfp8_grouped_gemm_x32_b200 import lib
    z = torch.zeros(1, dtype=torch.float32, device="cuda")
    lib.moe_router_topk(z.data_ptr(), lib.MOE_DTYPE_F32, 0, 8, 2, z.data_ptr(), z.data_ptr(), 0)
    torch.cuda.synchronize()
    assert float(z[0]) == 0.0


@pytest.mark.parametrize("name,T,training", [("qwen3_30b_ragged", 3000, True), ("tiny", 1000, False),
                                             ("gpt_oss_20b", 517, True)])
def test_route_permute_equals_router_then_permute(cuda, name, T, training):
    """moe_route_permute (the router fused into the permutation's histogram
    pass) writes exactly what moe_router_topk followed by moe_permute writes,
    and its expert ids match the oracle's router."""
    import torch
    from mxfp8_grouped_gemm_x32_b200.layer import GroupedMLP
    cfg = get_config(name, T=T)
    inp = make_inputs(cfg, seed=3, weights=False, grad=False)
    lg = torch.from_numpy(inp["router_logits"].astype(np.float32)).cuda()
    x = torch.from_numpy(inp["x"].view(np.int16)).view(torch.bfloat16).cuda()
    a = GroupedMLP(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, backward=training)
    b = GroupedMLP(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, backward=training)
    idx, prob = a.route(lg)
    a.permute(x, idx, prob, with_cols=training)
    b.route_permute(lg, x, with_cols=training)
    torch.cuda.synchronize()
    from mxfp8_grouped_gemm_x32_b200 import lib
    assert lib.moe_get_device_status(0) == 0
    ri, _ = orouter.route_topk(inp["router_logits"].astype(np.float32), cfg.k)
    assert np.array_equal(b.topk_idx.cpu().numpy(), ri)
    go = int(a.group_offsets[cfg.E])
    names = ["topk_idx", "topk_prob", "split_sizes", "group_offsets", "row_to_slot", "slot_to_row", "prob_perm"]
    for n in names:
        assert torch.equal(getattr(a, n), getattr(b, n)), n
    assert torch.equal(a.xq[: go * cfg.H], b.xq[: go * cfg.H])        # rows past the last group: unwritten
    nsf = lib.moe_mx_scale_bytes(1, go, cfg.H)
    assert torch.equal(a.xq_sf[:nsf], b.xq_sf[:nsf])
    if training:
        xa = a.xq_col[: cfg.H * a.rows_cap].view(cfg.H, a.rows_cap)[:, :go]
        xb = b.xq_col[: cfg.H * b.rows_cap].view(cfg.H, b.rows_cap)[:, :go]
        assert torch.equal(xa, xb)
