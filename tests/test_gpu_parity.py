"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bars: quantised bytes and scales bit-exact; index maps bit-exact;
requantised h and da: <= 1e-3 of elements differ, each by <= 1 E4M3 ulp
(scale differences only at oracle block maxima within 1e-5 of a scale
boundary); out: max|gpu - oracle| / rms(oracle) <= 2e-2; dX, dW1, dW2,
dprob: <= 3e-2 -- both after an element-wise allowance for requantised codes
whose oracle value sits on a rounding boundary within fp32 accuracy (either
code is correct there; tests/ambiguity.py derives it from oracle data only) --
and rms(gpu - oracle) / rms(oracle) <= 1e-2 with no allowance.
"""
import numpy as np
import pytest

from mxfp8_grouped_gemm_x32_b200.workloads import (bf16_bits_to_f32, get_config,
                                                   make_inputs)
from oracle import moe as omoe
from oracle import mxfp8 as omx

from . import ambiguity
from .mxutil import (bf16_to_f64, rel_max_over_rms, requant_mismatch, sf_padding_offsets,
                     sf_unblock)

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-2
GRAD_TOL = 3e-2
REQUANT_FRAC = 1e-3
RMS_TOL = 1e-2      # rms(gpu - oracle) / rms(oracle): every element, no allowance


def rel_rms(gpu, ref):
    return float(np.sqrt(np.mean((np.asarray(gpu) - ref) ** 2)) / np.sqrt(np.mean(ref ** 2)))


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mxfp8_grouped_gemm_x32_b200 import lib  # noqa: F401  (fails loudly if not built)
    return torch


def _bf(torch, bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _f64(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


def _special_matrix(rng, rows, cols):
    """bf16 test matrix: normals at per-row random scales, a zero block,
    tiny values, huge values and exact E4M3 ties."""
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    x *= np.exp2(rng.integers(-30, 30, (rows, 1))).astype(np.float32)
    x[0, :32] = 0.0
    x[1 % rows, :32] = np.float32(2.0 ** -130)
    x[2 % rows, 32:64] = np.float32(3.0e38)
    x[3 % rows, :32] = np.float32(448.0)
    x[3 % rows, 1] = np.float32(1.0625 * 256)     # tie between two codes at s = 0
    from mxfp8_grouped_gemm_x32_b200.workloads import bf16_bits_from_f32
    return bf16_bits_from_f32(x)


@pytest.mark.parametrize("groups,rows,cols", [(1, 256, 4096), (2, 200, 2880), (3, 64, 256)])
def test_quantize_rows_bitexact(torch_cuda, groups, rows, cols):
    torch = torch_cuda
    from mxfp8_grouped_gemm_x32_b200 import lib
    rng = np.random.default_rng(groups * 1000 + rows)
    bits = _special_matrix(rng, groups * rows, cols)
    src = _bf(torch, bits)
    q = torch.empty(groups * rows * cols, dtype=torch.uint8, device="cuda")
    nsf = lib.moe_mx_scale_bytes(groups, rows, cols)
    sf = torch.full((nsf,), 0xAB, dtype=torch.uint8, device="cuda")
    lib.moe_mlp_quantize_mxfp8(src.data_ptr(), groups, rows, cols, lib.MOE_QUANT_ROW, q.data_ptr(),
                               sf.data_ptr(), 0)
    torch.cuda.synchronize()
    c, s = omx.quantize_rows(_f64(bits))
    assert np.array_equal(q.cpu().numpy().reshape(groups * rows, cols), c)
    sfn = sf.cpu().numpy()
    assert np.array_equal(sf_unblock(sfn, groups, rows, cols).reshape(groups * rows, -1), s)
    assert np.all(sfn[sf_padding_offsets(groups, rows, cols)] == 0)


@pytest.mark.parametrize("groups,rows,cols", [(1, 384, 256), (2, 2880, 136), (4, 64, 2880)])
def test_quantize_cols_bitexact(torch_cuda, groups, rows, cols):
    torch = torch_cuda
    from mxfp8_grouped_gemm_x32_b200 import lib
    rng = np.random.default_rng(groups * 7 + cols)
    bits = _special_matrix(rng, groups * rows, cols)
    src = _bf(torch, bits)
    q = torch.empty(groups * rows * cols, dtype=torch.uint8, device="cuda")
    nsf = lib.moe_mx_scale_bytes(groups, cols, rows)
    sf = torch.full((nsf,), 0xAB, dtype=torch.uint8, device="cuda")
    lib.moe_mlp_quantize_mxfp8(src.data_ptr(), groups, rows, cols, lib.MOE_QUANT_COL, q.data_ptr(),
                               sf.data_ptr(), 0)
    torch.cuda.synchronize()
    qn = q.cpu().numpy().reshape(groups, cols, rows)
    sfu = sf_unblock(sf.cpu().numpy(), groups, cols, rows)
    x = _f64(bits).reshape(groups, rows, cols)
    for g in range(groups):
        c, s = omx.quantize_rows(x[g].T)
        assert np.array_equal(qn[g], c)
        assert np.array_equal(sfu[g], s)
    assert np.all(sf.cpu().numpy()[sf_padding_offsets(groups, cols, rows)] == 0)


class Layer:
    """Runs the CUDA layer on one workload and keeps host copies."""

    def __init__(self, torch, cfg, inp):
        from mxfp8_grouped_gemm_x32_b200.layer import GroupedMLP
        self.cfg, self.inp = cfg, inp
        # every buffer is followed by 4 KB of guard bytes (checked below)
        self.L = GroupedMLP(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, backward=True, guard=4096)
        self.args = (_bf(torch, inp["x"]), torch.from_numpy(inp["topk_idx"]).cuda(),
                     torch.from_numpy(inp["topk_prob"]).cuda(), _bf(torch, inp["w1"]),
                     _bf(torch, inp["w2"]), _bf(torch, inp["dy"]))
        self.res = self.L.step(*self.args)
        # the permutation once more with the optional column form of x (the
        # backward makes its own): checked in test_permute_bitexact
        self.L.permute(self.args[0], self.args[1], self.args[2], with_cols=True)
        torch.cuda.synchronize()
        from mxfp8_grouped_gemm_x32_b200 import lib
        self.status = lib.moe_get_device_status(0)


def _oracle(cfg, inp):
    x, w1, w2, dy = (_f64(inp[k]) for k in ("x", "w1", "w2", "dy"))
    f = omoe.forward(x, w1, w2, inp["topk_idx"], inp["topk_prob"])
    b = omoe.backward(f, x, w1, w2, inp["topk_prob"], dy)
    return f, b


def _padded_offsets(split):
    pad = (np.asarray(split) + 127) // 128 * 128
    return np.concatenate([[0], np.cumsum(pad)])


CASES = {
    "tiny": (dict(), None),
    "gptoss_k2880": (dict(name="gpt_oss_20b", T=160, E=4, k=2), None),
    "ragged_128e": (dict(name="qwen3_30b_ragged", T=96, H=256, I=256, E=128, k=8), None),
    "empty_and_single": (dict(T=200, E=6, k=1), "empty"),
    "all_on_one": (dict(T=300, E=4, k=2), "one"),
}


def _case(name):
    over, special = CASES[name]
    over = dict(over)
    base = over.pop("name", "tiny")
    cfg = get_config(base, **over)
    idx = None
    if special == "empty":
        rng = np.random.default_rng(5)
        idx = rng.choice([0, 2, 3, 5], size=(cfg.T, 1)).astype(np.int32)
        idx[17, 0] = 4                                   # expert 4: exactly one row; 1 empty
    elif special == "one":
        idx = np.stack([np.zeros(cfg.T, np.int32), np.full(cfg.T, 3, np.int32)], axis=1)
        idx[::7, 1] = 1
    inp = make_inputs(cfg, seed=11, topk_idx=idx)
    return cfg, inp


@pytest.fixture(scope="module", params=list(CASES))
def run(request, torch_cuda):
    cfg, inp = _case(request.param)
    layer = Layer(torch_cuda, cfg, inp)
    f, b = _oracle(cfg, inp)
    x, w1, w2, dy = (_f64(inp[k]) for k in ("x", "w1", "w2", "dy"))
    allow = ambiguity.backward_allowance(f, b, x, w1, w2, dy, inp["topk_idx"])
    allow["out"] = ambiguity.forward_allowance(f, x, w1, w2, inp["topk_idx"])
    f["allow"] = allow
    return cfg, inp, layer, f, b


def test_device_status_clean(run):
    cfg, inp, layer, f, b = run
    assert layer.status == 0


def test_no_write_past_any_buffer(run):
    """The guard bytes after every output and workspace buffer of the step
    (weights, routing, activations, gradients, workspaces) are intact."""
    cfg, inp, layer, f, b = run
    assert layer.L.check_guards() == []


def test_permute_bitexact(run):
    cfg, inp, layer, f, b = run
    L = layer.L
    split = L.split_sizes.cpu().numpy()
    go = L.group_offsets.cpu().numpy()
    assert np.array_equal(split, f["split_sizes"])
    assert np.array_equal(go, _padded_offsets(split))
    r2s = L.row_to_slot.cpu().numpy()
    s2r = L.slot_to_row.cpu().numpy()
    pp = L.prob_perm.cpu().numpy()
    offs = f["offsets"]
    xq = L.xq.cpu().numpy()[: L.rows_cap * cfg.H].reshape(L.rows_cap, cfg.H)
    xsf = sf_unblock(L.xq_sf.cpu().numpy(), 1, L.rows_cap, cfg.H)[0]
    xcol = L.xq_col.cpu().numpy()[: cfg.H * L.rows_cap].reshape(cfg.H, L.rows_cap)
    xcsf = sf_unblock(L.xq_col_sf.cpu().numpy(), 1, cfg.H, L.rows_cap)[0]
    x = _f64(inp["x"])
    used = np.zeros(L.rows_cap, bool)
    for e in range(cfg.E):
        g0, n = go[e], split[e]
        rows = slice(g0, g0 + n)
        used[rows] = True
        assert np.array_equal(r2s[rows], f["perm"][offs[e]:offs[e + 1]])
        assert np.array_equal(xq[rows], f["xq_codes"][offs[e]:offs[e + 1]])
        assert np.array_equal(xsf[rows], f["xq_scales"][offs[e]:offs[e + 1]])
        assert np.array_equal(pp[rows], inp["topk_prob"].reshape(-1)[f["perm"][offs[e]:offs[e + 1]]])
        # along tokens, blocks restart at the group start
        c, s = omx.quantize_cols_grouped(x[f["tok"][offs[e]:offs[e + 1]]], [n])[0]
        mp = c.shape[1]
        assert np.array_equal(xcol[:, g0:g0 + mp], c)
        assert np.array_equal(xcsf[:, g0 // 32:(g0 + mp) // 32], s)
        assert np.all(xcol[:, g0 + mp:go[e + 1]] == 0)
    assert np.all(r2s[~used] == -1)
    pad = ~used[: go[cfg.E]]        # padding rows inside the groups (rows past the last group are not written)
    assert np.all(xq[: go[cfg.E]][pad] == 0) and np.all(xsf[: go[cfg.E]][pad] == 0)

    assert np.array_equal(s2r[r2s[used]], np.flatnonzero(used))
    assert np.all(pp[~used] == 0)


def test_forward_requant_and_saved(run):
    cfg, inp, layer, f, b = run
    L = layer.L
    go = L.group_offsets.cpu().numpy()
    split = f["split_sizes"]
    offs = f["offsets"]
    sel = np.concatenate([np.arange(go[e], go[e] + split[e]) for e in range(cfg.E)]).astype(np.int64)
    hq = L.hq.cpu().numpy()[: L.rows_cap * cfg.I].reshape(L.rows_cap, cfg.I)[sel]
    hsf = sf_unblock(L.hq_sf.cpu().numpy(), 1, L.rows_cap, cfg.I)[0][sel]
    # oracle block amax of h (unrounded) for the scale-boundary allowance
    A = f["A"]
    h = f["p"][:, None] * omoe.silu(A[:, :cfg.I]) * A[:, cfg.I:]
    amax = np.abs(h).reshape(h.shape[0], -1, 32).max(axis=2)
    frac, max_ulp, bad = requant_mismatch(hq, hsf, f["hq_codes"], f["hq_scales"], amax)
    assert frac <= REQUANT_FRAC, frac
    assert max_ulp <= 1
    assert bad == 0
    # saved activation: bf16 of A on both sides; where A's accumulation band
    # spans a bf16 rounding boundary, any bf16 value inside the band is right
    saved = bf16_to_f64(L.saved_a)[sel]
    ref = f["saved"]
    x, w1 = _f64(inp["x"]), _f64(inp["w1"])
    ok = saved == ref
    for e in range(cfg.E):
        sl = slice(offs[e], offs[e + 1])
        if sl.stop == sl.start:
            continue
        band = ambiguity.acc_band(omx.roundtrip_rows(x[f["tok"][sl]]), omx.roundtrip_rows(w1[e]))
        lo, hi = ambiguity.bf16_alternatives(f["A"][sl], band)
        ok[sl] |= (saved[sl] >= lo) & (saved[sl] <= hi)
    assert np.all(ok), np.argwhere(~ok)[:5]
    assert np.mean(saved != ref) <= REQUANT_FRAC


def test_forward_output(run):
    cfg, inp, layer, f, b = run
    out = bf16_to_f64(layer.res[0])
    # max |gpu - oracle| / rms(oracle), after the allowance for requantised
    # codes that sit on a rounding boundary within fp32 accuracy
    assert ambiguity.within(out, f["out"], OUT_TOL, f["allow"]["out"]) <= OUT_TOL
    assert rel_rms(out, f["out"]) <= RMS_TOL


@pytest.mark.parametrize("key,ref", [("dX", "dX"), ("dW1", "dW1"), ("dW2", "dW2"), ("dprob", "dprob_f64")])
def test_backward_outputs(run, key, ref):
    cfg, inp, layer, f, b = run
    i = {"dX": 1, "dW1": 2, "dW2": 3, "dprob": 4}[key]
    gpu = layer.res[i]
    g = gpu.float().cpu().numpy().astype(np.float64)
    assert ambiguity.within(g, b[ref], GRAD_TOL, f["allow"][key], bf16_out=key != "dprob") <= GRAD_TOL
    assert rel_rms(g, b[ref]) <= RMS_TOL
    if key in ("dW1", "dW2"):
        empty = np.flatnonzero(f["split_sizes"] == 0)
        assert np.all(g[empty] == 0)


def test_backward_requant_da(run):
    """da = [dg | du] requantised along 2I matches the oracle's codec applied
    to the oracle's da (read from the backward workspace)."""
    cfg, inp, layer, f, b = run
    # the row-quantised da lives in the backward workspace: see carve_bwd
    # (dyq, dyq_sf, dyc, dyc_sf, daq, ...), 256-byte aligned pieces
    L = layer.L
    rc, H, I = L.rows_cap, cfg.H, cfg.I
    from mxfp8_grouped_gemm_x32_b200 import lib
    a256 = lambda n: (n + 255) // 256 * 256
    off = (a256(rc * H) + a256(lib.moe_mx_scale_bytes(1, rc, H)) + a256(H * rc)
           + a256(lib.moe_mx_scale_bytes(1, H, rc)))
    ws = L.ws_bwd.cpu().numpy()
    daq = ws[off:off + rc * 2 * I].reshape(rc, 2 * I)
    off2 = off + a256(rc * 2 * I)
    dasf = sf_unblock(ws[off2:off2 + lib.moe_mx_scale_bytes(1, rc, 2 * I)], 1, rc, 2 * I)[0]
    go = L.group_offsets.cpu().numpy()
    split = f["split_sizes"]
    sel = np.concatenate([np.arange(go[e], go[e] + split[e]) for e in range(cfg.E)]).astype(np.int64)
    c, s = omx.quantize_rows(b["da"])
    amax = np.abs(b["da"]).reshape(b["da"].shape[0], -1, 32).max(axis=2)
    frac, max_ulp, bad = requant_mismatch(daq[sel], dasf[sel], c, s, amax)
    assert frac <= REQUANT_FRAC, frac
    assert max_ulp <= 1
    assert bad == 0


def test_backward_dy_codes_bitexact(run):
    """dY gathered to permuted rows and quantised along H and along tokens (the
    backward workspace's first four pieces: see carve_bwd) equals the oracle's
    codec on the gathered rows, bit for bit; padding rows are zero."""
    cfg, inp, layer, f, b = run
    L = layer.L
    rc, H = L.rows_cap, cfg.H
    from mxfp8_grouped_gemm_x32_b200 import lib
    a256 = lambda n: (n + 255) // 256 * 256
    ws = L.ws_bwd.cpu().numpy()
    o_sf = a256(rc * H)
    o_c = o_sf + a256(lib.moe_mx_scale_bytes(1, rc, H))
    o_csf = o_c + a256(H * rc)
    dyq = ws[:rc * H].reshape(rc, H)
    dysf = sf_unblock(ws[o_sf:o_sf + lib.moe_mx_scale_bytes(1, rc, H)], 1, rc, H)[0]
    dyc = ws[o_c:o_c + H * rc].reshape(H, rc)
    dycsf = sf_unblock(ws[o_csf:o_csf + lib.moe_mx_scale_bytes(1, H, rc)], 1, H, rc)[0]
    dy = _f64(inp["dy"])
    go = L.group_offsets.cpu().numpy()
    offs = f["offsets"]
    for e in range(cfg.E):
        g0, n = go[e], f["split_sizes"][e]
        tok = f["tok"][offs[e]:offs[e + 1]]
        c, s = omx.quantize_rows(dy[tok])
        assert np.array_equal(dyq[g0:g0 + n], c) and np.array_equal(dysf[g0:g0 + n], s)
        assert np.all(dyq[g0 + n:go[e + 1]] == 0) and np.all(dysf[g0 + n:go[e + 1]] == 0)
        c, s = omx.quantize_cols_grouped(dy[tok], [n])[0]
        mp = c.shape[1]
        assert np.array_equal(dyc[:, g0:g0 + mp], c)
        assert np.array_equal(dycsf[:, g0 // 32:(g0 + mp) // 32], s)
        assert np.all(dyc[:, g0 + mp:go[e + 1]] == 0)


def test_wait_timeout_selftest(torch_cuda):
    from mxfp8_grouped_gemm_x32_b200 import lib
    st = lib.moe_selftest_wait_timeout(20, 0)
    assert st == 6, lib.status_string(st)          # MOE_ERR_TIMEOUT
    assert lib.moe_get_device_status(0) == 0       # read-and-clear


def test_bad_expert_id_reported(torch_cuda):
    torch = torch_cuda
    from mxfp8_grouped_gemm_x32_b200.layer import GroupedMLP
    from mxfp8_grouped_gemm_x32_b200 import lib
    cfg = get_config("tiny", T=64)
    inp = make_inputs(cfg, seed=2)
    idx = inp["topk_idx"].copy()
    idx[3, 1] = cfg.E + 5
    L = GroupedMLP(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, backward=False)
    L.permute(_bf(torch, inp["x"]), torch.from_numpy(idx).cuda(), torch.from_numpy(inp["topk_prob"]).cuda())
    assert lib.moe_get_device_status(0) == 5       # MOE_ERR_DEVICE_INDEX
    assert L.slot_to_row.cpu().numpy()[3 * cfg.k + 1] == -1


@pytest.mark.parametrize("E,H,I", [(3, 256, 192), (2, 2880, 2880), (2, 4096, 512)])
def test_quantize_weights_fused_equals_separate(torch_cuda, E, H, I):
    """moe_mlp_quantize_weights (one read of each weight) writes exactly what
    the four single-mode calls write, including zero padding scale bytes."""
    torch = torch_cuda
    from mxfp8_grouped_gemm_x32_b200 import lib
    rng = np.random.default_rng(E * H + I)
    from mxfp8_grouped_gemm_x32_b200.workloads import bf16_bits_from_f32
    w1 = _bf(torch, bf16_bits_from_f32(rng.standard_normal((E, 2 * I, H)).astype(np.float32) * 0.05))
    w2 = _bf(torch, bf16_bits_from_f32(rng.standard_normal((E, H, I)).astype(np.float32) * 0.05))
    sb = lib.moe_mx_scale_bytes
    sizes = [(2 * E * I * H, sb(2 * E, I, H)), (E * H * I, sb(E, H, I)), (E * H * 2 * I, sb(E, H, 2 * I)),
             (E * I * H, sb(E, I, H))]

    def bufs():
        return [(torch.full((q,), 0x33, dtype=torch.uint8, device="cuda"),
                 torch.full((s,), 0x33, dtype=torch.uint8, device="cuda")) for q, s in sizes]
    a, b = bufs(), bufs()
    p = lambda t: t.data_ptr()
    lib.moe_mlp_quantize_mxfp8(p(w1), 2 * E, I, H, lib.MOE_QUANT_ROW, p(a[0][0]), p(a[0][1]), 0)
    lib.moe_mlp_quantize_mxfp8(p(w2), E, H, I, lib.MOE_QUANT_ROW, p(a[1][0]), p(a[1][1]), 0)
    lib.moe_mlp_quantize_mxfp8(p(w1), E, 2 * I, H, lib.MOE_QUANT_COL, p(a[2][0]), p(a[2][1]), 0)
    lib.moe_mlp_quantize_mxfp8(p(w2), E, H, I, lib.MOE_QUANT_COL, p(a[3][0]), p(a[3][1]), 0)
    lib.moe_mlp_quantize_weights(p(w1), p(w2), E, H, I, p(b[0][0]), p(b[0][1]), p(b[1][0]), p(b[1][1]),
                                 p(b[2][0]), p(b[2][1]), p(b[3][0]), p(b[3][1]), 0)
    torch.cuda.synchronize()
    for (qa, sa), (qb, sb_) in zip(a, b):
        assert torch.equal(qa, qb) and torch.equal(sa, sb_)
    # and against the oracle for the forward operands
    c, s = omx.quantize_rows(_f64(w1.cpu().view(torch.int16).numpy().view(np.uint16)).reshape(2 * E * I, H))
    assert np.array_equal(b[0][0].cpu().numpy().reshape(2 * E * I, H), c)
    assert np.array_equal(sf_unblock(b[0][1].cpu().numpy(), 2 * E, I, H).reshape(2 * E * I, -1), s)


@pytest.mark.parametrize("T", [0, 1])
def test_zero_and_one_token(torch_cuda, T):
    """A batch with no tokens runs every launch of the step and leaves nothing
    to compute (zero weight gradients); a single token is one row in each of
    its k experts' groups."""
    import torch
    from mxfp8_grouped_gemm_x32_b200 import lib
    from mxfp8_grouped_gemm_x32_b200.layer import GroupedMLP
    cfg = get_config("tiny", T=T)
    inp = make_inputs(cfg, seed=3)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    L = GroupedMLP(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    res = L.step(bf(inp["x"]), torch.from_numpy(inp["topk_idx"]).cuda(), torch.from_numpy(inp["topk_prob"]).cuda(),
                 bf(inp["w1"]), bf(inp["w2"]), bf(inp["dy"]))
    torch.cuda.synchronize()
    assert lib.moe_get_device_status(0) == 0
    out, dX, dW1, dW2, dprob = res
    assert out.shape == (T, cfg.H) and dprob.shape == (T, cfg.k)
    if T == 0:
        assert float(dW1.float().abs().max()) == 0.0 and float(dW2.float().abs().max()) == 0.0
        return
    f = omoe.forward(_f64(inp["x"]), _f64(inp["w1"]), _f64(inp["w2"]), inp["topk_idx"], inp["topk_prob"])
    b = omoe.backward(f, _f64(inp["x"]), _f64(inp["w1"]), _f64(inp["w2"]), inp["topk_prob"], _f64(inp["dy"]))
    x, w1, w2, dy = (_f64(inp[k]) for k in ("x", "w1", "w2", "dy"))
    allow = ambiguity.backward_allowance(f, b, x, w1, w2, dy, inp["topk_idx"])
    allow["out"] = ambiguity.forward_allowance(f, x, w1, w2, inp["topk_idx"])
    assert ambiguity.within(bf16_to_f64(out), f["out"], OUT_TOL, allow["out"]) <= OUT_TOL
    for key, gpu, ref, bfo in (("dX", dX, b["dX"], True), ("dprob", dprob, b["dprob_f64"], False)):
        g = gpu.float().cpu().numpy().astype(np.float64)
        assert ambiguity.within(g, ref, GRAD_TOL, allow[key], bf16_out=bfo) <= GRAD_TOL


@pytest.mark.parametrize("name,over", [("tiny", {}), ("gpt_oss_20b", dict(T=160, E=4, k=2))])
def test_forward_only_equals_training_forward(torch_cuda, name, over):
    """The inference path (permutation quantising x along H only, forward
    without the saved activation) writes exactly the bytes of the training
    path's permutation and forward."""
    torch = torch_cuda
    from mxfp8_grouped_gemm_x32_b200 import lib
    from mxfp8_grouped_gemm_x32_b200.layer import GroupedMLP
    cfg = get_config(name, **over)
    inp = make_inputs(cfg, seed=4, grad=False)
    x, w1, w2 = (_bf(torch, inp[k]) for k in ("x", "w1", "w2"))
    idx, prob = torch.from_numpy(inp["topk_idx"]).cuda(), torch.from_numpy(inp["topk_prob"]).cuda()
    outs = []
    for bwd in (False, True):
        L = GroupedMLP(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, backward=bwd)
        L.quantize_weights(w1, w2)
        L.permute(x, idx, prob)
        out = L.forward()
        torch.cuda.synchronize()
        routed = L.row_to_slot.cpu().numpy() >= 0    # h is written for routed rows only
        rc = L.rows_cap
        h = L.hq.cpu().numpy()[: rc * cfg.I].reshape(rc, cfg.I)[routed]
        hs = sf_unblock(L.hq_sf.cpu().numpy(), 1, rc, cfg.I)[0][routed]
        used = int(L.group_offsets[cfg.E])           # rows past the last group are not written
        xq = L.xq.cpu().numpy()[: used * cfg.H]
        xs = L.xq_sf.cpu().numpy()[: lib.moe_mx_scale_bytes(1, used, cfg.H)]
        outs.append([xq, xs, h, hs, out.view(torch.uint8).cpu().numpy()])
    for a, b in zip(*outs):
        assert np.array_equal(a, b)
