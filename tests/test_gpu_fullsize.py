"""Full-size parity on sampled outputs: the Mixtral-8x7B, Qwen3-30B-shaped
(128 experts, skewed routing) and GPT-OSS-20B-shaped layers at their real
sizes, run through the same layer object and launch sequence bench.py times
(weight quantisation, permute, forward, backward).

The oracle cannot run the whole layer in float64 in seconds, so it checks
samples through sub-problems that reproduce the full layer's arithmetic for
the sampled outputs exactly (every row's forward and backward depend only on
that row and its expert's weights; every intermediate channel's weight
gradients depend only on that channel over the expert's rows, with the same
32-row blocks along tokens):
* for three experts -- the median, the largest (many 128-row tiles) and the
  smallest non-empty group: per-slot outputs of a few routed rows including
  the group's first and last (the down-projection row y and the dgrad row dx,
  fp32 before the combine, and dprob), and two 32-channel blocks of the
  expert's weight gradients, one of them the last (dW_gate_up rows, gate and
  up, and dW_down columns) over every routed row of the expert;
* at every token: out = bf16(sum_j y) and dX = bf16(sum_j dx), bit-exact, with
  y and dx the f24 rows the library keeps (the combine, a property that holds
  at any size).
Bars as in test_gpu_parity.py (with the allowance of tests/ambiguity.py).
"""
import numpy as np
import pytest

from mxfp8_grouped_gemm_x32_b200.workloads import (bf16_bits_from_f32, bf16_bits_to_f32, get_config,
                                                   make_inputs)
from oracle import moe as omoe

from . import ambiguity

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

OUT_TOL, GRAD_TOL, RMS_TOL = 2e-2, 3e-2, 1e-2


def _f64(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


def _rel_rms(g, r):
    return float(np.sqrt(np.mean((g - r) ** 2)) / np.sqrt(np.mean(r ** 2)))


def _slot_buffers(L, cfg):
    """Rows kept by the library in the caller's workspaces: the forward's y
    (first piece when hq is caller-provided) and the backward's dx (the piece
    after the MX operands), both [rows_cap][H] f24 rows in permuted order,
    returned as float32 in slot order."""
    import torch
    from mxfp8_grouped_gemm_x32_b200 import lib
    rc, H, I = L.rows_cap, cfg.H, cfg.I
    a256 = lambda v: (v + 255) // 256 * 256
    sb = lib.moe_mx_scale_bytes
    pieces = [rc * H, sb(1, rc, H), H * rc, sb(1, H, rc), rc * 2 * I, sb(1, rc, 2 * I),
              2 * I * rc, sb(1, 2 * I, rc), I * rc, sb(1, I, rc)]
    off = sum(a256(p) for p in pieces)
    s2r = L.slot_to_row.cpu().numpy().astype(np.int64)
    y = _f24_rows(L.ws_fwd[: rc * H * 3], rc, H)
    dx = _f24_rows(L.ws_bwd[off: off + rc * H * 3], rc, H)
    return torch.from_numpy(y[s2r]).cuda(), torch.from_numpy(dx[s2r]).cuda()


def _f24_rows(buf, rows, H):
    """Rows stored as f24 (the top 24 bits of each fp32 value, 3 bytes per
    value, little-endian) -> float32 [rows, H]."""
    b = buf.cpu().numpy().reshape(rows, H, 3).astype(np.uint32)
    bits = (b[..., 0] << np.uint32(8)) | (b[..., 1] << np.uint32(16)) | (b[..., 2] << np.uint32(24))
    return bits.view(np.float32)


@pytest.mark.parametrize("name", ["mixtral_8x7b", "qwen3_30b_ragged", "gpt_oss_20b"])
def test_full_size_sampled(name):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mxfp8_grouped_gemm_x32_b200 import lib
    from mxfp8_grouped_gemm_x32_b200.layer import GroupedMLP

    cfg = get_config(name)
    inp = make_inputs(cfg, seed=0)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    L = GroupedMLP(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    out, dX, dW1, dW2, dprob = L.step(bf(inp["x"]), torch.from_numpy(inp["topk_idx"]).cuda(),
                                      torch.from_numpy(inp["topk_prob"]).cuda(), bf(inp["w1"]),
                                      bf(inp["w2"]), bf(inp["dy"]))
    torch.cuda.synchronize()
    assert lib.moe_get_device_status(0) == 0
    idx, prob = inp["topk_idx"], inp["topk_prob"]
    split = np.bincount(idx.reshape(-1), minlength=cfg.E)
    assert np.array_equal(L.split_sizes.cpu().numpy(), split)

    # --- combine at every token: out = bf16(sum_j y[t*k+j]) (fp32, j ascending)
    y_slot, dx_slot = _slot_buffers(L, cfg)
    for gpu_sum, rows in ((out, y_slot), (dX, dx_slot)):
        r = rows.cpu().numpy().reshape(cfg.T, cfg.k, cfg.H)
        acc = r[:, 0].copy()
        for j in range(1, cfg.k):
            acc = (acc + r[:, j]).astype(np.float32)
        want = bf16_bits_from_f32(acc)
        got = gpu_sum.cpu().view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(got, want)

    # --- three experts: the median, the largest and the smallest non-empty
    # group (the largest spans many 128-row tiles; every group has a ragged
    # last tile, and on the GPT-OSS shape both contractions end in a K tail)
    nz = np.flatnonzero(split)
    order = nz[np.argsort(split[nz], kind="stable")]
    experts = []
    for e in (int(order[len(order) // 2]), int(order[-1]), int(order[0])):
        if e not in experts:
            experts.append(e)
    x = _f64(inp["x"])
    dy = _f64(inp["dy"])
    for n, e in enumerate(experts):
        _check_expert(cfg, inp, L, e, x, dy, y_slot, dx_slot, dW1, dW2, dprob, seed=1 + n)


def _check_expert(cfg, inp, L, e, x, dy, y_slot, dx_slot, dW1, dW2, dprob, seed):
    import torch
    idx, prob = inp["topk_idx"], inp["topk_prob"]
    slots = np.flatnonzero(idx.reshape(-1) == e)          # its rows, in permuted (slot) order
    tk = slots // cfg.k
    pe = prob.reshape(-1)[slots][:, None].astype(np.float32)
    w1e = _f64(inp["w1"][e:e + 1])
    w2e = _f64(inp["w2"][e:e + 1])
    rng = np.random.default_rng(seed)

    # sampled rows: y, dx, dprob (k = 1 sub-problem over those rows); the
    # group's first and last rows are always among them
    pick = rng.choice(slots.size, min(8, slots.size), replace=False)
    s = np.unique(np.concatenate([pick, [0, slots.size - 1]]))
    xs, dys = x[tk[s]], dy[tk[s]]
    i1 = np.zeros((s.size, 1), np.int32)
    f = omoe.forward(xs, w1e, w2e, i1, pe[s])
    b = omoe.backward(f, xs, w1e, w2e, pe[s], dys)
    a_y = ambiguity.forward_allowance(f, xs, w1e, w2e, i1)
    a_b = ambiguity.backward_allowance(f, b, xs, w1e, w2e, dys, i1)
    g_y = y_slot[torch.from_numpy(slots[s]).cuda()].cpu().numpy().astype(np.float64)
    g_dx = dx_slot[torch.from_numpy(slots[s]).cuda()].cpu().numpy().astype(np.float64)
    g_dp = dprob.reshape(-1)[torch.from_numpy(slots[s]).cuda()].cpu().numpy().astype(np.float64)
    tag = f"expert {e} ({slots.size} rows)"
    assert ambiguity.within(g_y, f["Y"], OUT_TOL, a_y, bf16_out=False) <= OUT_TOL, tag
    assert ambiguity.within(g_dx, b["dx_rows"], GRAD_TOL, a_b["dX"], bf16_out=False) <= GRAD_TOL, tag
    assert ambiguity.within(g_dp, b["dprob_f64"][:, 0], GRAD_TOL, a_b["dprob"][:, 0], bf16_out=False) <= GRAD_TOL, tag
    assert _rel_rms(g_y, f["Y"]) <= RMS_TOL and _rel_rms(g_dx, b["dx_rows"]) <= RMS_TOL, tag

    # two 32-channel blocks of the intermediate dimension (one of them the
    # last block), over all rows of e
    I = cfg.I
    blocks = np.unique([rng.integers(0, I // 32 - 1), I // 32 - 1])
    ch = np.concatenate([np.arange(32 * c, 32 * c + 32) for c in blocks])
    w1c = np.concatenate([w1e[:, ch], w1e[:, I + ch]], axis=1)      # [1, 2*nch, H]
    w2c = w2e[:, :, ch]                                              # [1, H, nch]
    ie = np.zeros((slots.size, 1), np.int32)
    fe = omoe.forward(x[tk], w1c, w2c, ie, pe)
    be = omoe.backward(fe, x[tk], w1c, w2c, pe, dy[tk])
    ae = ambiguity.backward_allowance(fe, be, x[tk], w1c, w2c, dy[tk], ie)
    rows1 = torch.from_numpy(np.concatenate([ch, I + ch])).cuda()
    g_w1 = dW1[e][rows1].float().cpu().numpy().astype(np.float64)
    g_w2 = dW2[e][:, torch.from_numpy(ch).cuda()].float().cpu().numpy().astype(np.float64)
    assert ambiguity.within(g_w1, be["dW1"][0], GRAD_TOL, ae["dW1"][0]) <= GRAD_TOL, tag
    assert ambiguity.within(g_w2, be["dW2"][0], GRAD_TOL, ae["dW2"][0]) <= GRAD_TOL, tag
    assert _rel_rms(g_w1, be["dW1"][0]) <= RMS_TOL and _rel_rms(g_w2, be["dW2"][0]) <= RMS_TOL, tag
