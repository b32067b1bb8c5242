#!/usr/bin/env python
"""Benchmark of the grouped MXFP8 MoE expert MLP (forward + backward).

One step = one pass of the whole hot path over one batch: weight
quantisation (both directions), permutation + quantisation of x, the fused
forward (gate_up GEMM + ScaledSwiGLU + requant, down GEMM, top-k combine)
and the backward (dY quantisation, dgrad / wgrad of both projections,
ScaledSwiGLU backward).  Metric: algorithmic TFLOP/s = 18 * R * H * I / step
time (R = T * k routed rows), and its fraction of the dense MXFP8 peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

Multi-GPU (torchrun, one process per GPU): every rank runs an independent
replica of the layer on its own batch (data-parallel tokens, weak scaling,
no collective on the data path); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mxfp8_grouped_gemm_x32_b200.workloads import get_config  # noqa: E402

METRIC = "grouped MoE MLP fwd/bwd TFLOP/s on 1 B200 and % of dense MXFP8 peak"
SIDE_WORKLOADS_DEFAULT = ("qwen3_30b_ragged", "gpt_oss_20b")
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0
MXFP8_OVER_BF16 = 2.0       # nominal dense ratio (4.5 / 2.25 PFLOP/s)
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "gemm_gate_up_swiglu.mixtral_8x7b.md")
GEMM_SOURCES = ["mxfp8_grouped_gemm_x32_b200/csrc/gemm.cu", "mxfp8_grouped_gemm_x32_b200/csrc/gemm.cuh",
                "mxfp8_grouped_gemm_x32_b200/csrc/common.cuh"]


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="mixtral_8x7b")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workloads", default=",".join(SIDE_WORKLOADS_DEFAULT),
                    help="further layer shapes measured in the same run (comma list; 'none' for none)")
    ap.add_argument("--no-library-probe", action="store_true",
                    help="skip the dense MXFP8 GEMM rate of the CUDA library (context for the roofline)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# host helpers (no GPU needed; covered by tests/test_bench_host.py)
# ---------------------------------------------------------------------------

def step_flops(cfg) -> float:
    """Algorithmic FLOPs of one forward + backward step (6RHI + 12RHI)."""
    return cfg.fwd_flops() + cfg.bwd_flops()


def gate_up_flops(cfg) -> float:
    """Algorithmic FLOPs of one launch of the gate_up GEMM: 2 * R * H * 2I."""
    return 4.0 * cfg.R * cfg.H * cfg.I


def bandwidth_bytes(cfg) -> dict:
    """Algorithmic HBM bytes per step of the bandwidth-bound kernels (reads
    + writes; MX codes count 1 byte and their scales 1/32 byte per value;
    x and dY are counted once per token however often they are gathered):
      quant_weights  bf16 W_gate_up and W_down in, both MX forms out;
      permute_quant  x in, R = T*k MX rows along H out;
      dy_quant       dY in, R rows along H and along tokens out;
      x_quant_cols   x in, R rows along tokens out;
      combine(_dx)   R f24 rows in (3 bytes per value), T bf16 rows out."""
    T, H, I, E, R = cfg.T, cfg.H, cfg.I, cfg.E, cfg.R
    mx = 1 + 1 / 32
    return {"quant_weights": 3.0 * E * H * I * (2 + 2 * mx),
            "permute_quant": T * H * 2 + R * H * mx,
            "dy_quant": T * H * 2 + 2 * R * H * mx,
            "x_quant_cols": T * H * 2 + R * H * mx,
            "combine": R * H * 3 + T * H * 2,
            "combine_dx": R * H * 3 + T * H * 2}


def annotate_bandwidth(kernels: dict, cfg, hbm_gbs: float) -> dict:
    """Adds algorithmic bytes per step, GB/s and the fraction of the HBM copy
    bandwidth to the bandwidth-bound kernels' entries."""
    for name, b in bandwidth_bytes(cfg).items():
        k = kernels.get(name)
        if k and k.get("ms_per_step"):
            gbs = b / (k["ms_per_step"] * 1e-3) / 1e9
            k.update({"bytes_per_step": b, "gbs": gbs, "frac_of_hbm": gbs / hbm_gbs})
    return kernels


L2_BYTES = 126 * 2 ** 20


def l2_note(cfg) -> str:
    """How the timed steps avoid L2 reuse between iterations: every step
    re-reads all bf16 master weights (3*E*H*I elements), which for the
    benchmarked layers is far more than the 126 MB L2."""
    wb = 3.0 * cfg.E * cfg.H * cfg.I * 2
    if wb > L2_BYTES:
        return f"inputs larger than L2 (bf16 weights {wb / 1e9:.2f} GB re-read each step)"
    return f"inputs smaller than L2 (bf16 weights {wb / 1e6:.1f} MB; no flush between steps)"


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over the process group (the step time of a
    multi-GPU run is the slowest rank's)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks(path=os.path.join(ROOT, "MEASURED_PEAKS.json")):
    """Dense MXFP8 peak (TFLOP/s) and HBM (GB/s) with the source named."""
    try:
        with open(path) as fh:
            p = json.load(fh)
        bf16 = float(p["bf16_tflops"])
        bf16_s = float(p.get("bf16_tflops_sustained", bf16))
        return {"mxfp8_burst": bf16 * MXFP8_OVER_BF16, "mxfp8_sustained": bf16_s * MXFP8_OVER_BF16,
                "bf16_sustained": bf16_s, "hbm_gbs": float(p["hbm_gbs"]), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"mxfp8_burst": FALLBACK_BF16_TFLOPS * MXFP8_OVER_BF16,
                "mxfp8_sustained": 1400.0 * MXFP8_OVER_BF16, "bf16_sustained": 1400.0,
                "hbm_gbs": FALLBACK_HBM_GBS, "source": "fallback"}


def mxfp8_library_probe(torch, dev, seconds: float = 3.0):
    """Dense MXFP8 GEMM rate of the CUDA library on this GPU (torch scaled_mm,
    1x32 block scales, 8192^3): best of 10 (burst) and a seconds-long loop
    (sustained, under the power cap).  Context for the roofline only -- it is
    not on the measured path.  None when the library does not offer it."""
    try:
        import torch.nn.functional as F
        M = N = K = 8192
        a = torch.randn(M, K, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn(N, K, device=dev).to(torch.float8_e4m3fn)
        sa = torch.full((M * K // 32,), 127, dtype=torch.uint8, device=dev).view(torch.float8_e8m0fnu)
        sb = torch.full((N * K // 32,), 127, dtype=torch.uint8, device=dev).view(torch.float8_e8m0fnu)
        bw, sw = F.ScalingType.BlockWise1x32, F.SwizzleType.SWIZZLE_32_4_4

        def run():
            return F.scaled_mm(a, b.t(), sa, bw, sb, bw, swizzle_a=sw, swizzle_b=sw, output_dtype=torch.bfloat16)
        run()
        torch.cuda.synchronize()
        best = float("inf")
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(10):
            e0.record()
            run()
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        n, t0 = 0, time.time()
        e0.record()
        while time.time() - t0 < seconds:
            for _ in range(20):
                run()
            n += 20
            torch.cuda.synchronize()
        e1.record()
        torch.cuda.synchronize()
        fl = 2.0 * M * N * K
        return {"what": "torch scaled_mm (cuBLAS) dense MXFP8 8192^3, 1x32 E8M0 scales",
                "burst_tflops": fl / best / 1e9, "sustained_tflops": fl / (e0.elapsed_time(e1) / n) / 1e9}
    except Exception as exc:  # library without MXFP8 scaled_mm
        return {"unavailable": f"{type(exc).__name__}: {exc}"[:200]}


def attainable_fwd(cfg, split, p_tflops: float, bw_gbs: float, rows_cap: int) -> dict:
    """Attainable layer-forward time: per expert e, max(FLOP_e / P, bytes_e / BW)
    for each of the two GEMMs (tiny groups are bound by their weight bytes),
    plus the permutation's and the combine's bytes at BW.  Bytes per GEMM:
    MX weights (+1/32 scales) and the expert's activation rows in and out
    (gate_up: x codes in, bf16 saved A and h codes out; down: h codes in,
    f24 rows out, 3 bytes per value)."""
    H, I, T, k = cfg.H, cfg.I, cfg.T, cfg.k
    P, BW = p_tflops * 1e12, bw_gbs * 1e9
    t = 0.0
    for m in split:
        m = float(m)
        f1, f2 = 2 * m * H * 2 * I, 2 * m * I * H
        b1 = 2 * I * H * (1 + 1 / 32) + m * H + m * 2 * I * 2 + m * I
        b2 = H * I * (1 + 1 / 32) + m * I + m * H * 3
        t += max(f1 / P, b1 / BW) + max(f2 / P, b2 / BW)
    permute_bytes = T * H * 2 + T * k * H * (1 + 1 / 32)
    combine_bytes = T * k * H * 3 + T * H * 2
    t += (permute_bytes + combine_bytes) / BW
    return {"ms": t * 1e3, "peak_tflops": p_tflops, "hbm_gbs": bw_gbs,
            "what": "sum over experts of max(FLOP/P, bytes/BW) for both GEMMs + permutation and combine bytes / BW"}


def split_histogram(split) -> dict:
    """Rows per expert (M_e) of one routing: min, median, max, and the number
    of experts that received no token."""
    m = sorted(int(v) for v in split)
    n = len(m)
    med = m[n // 2] if n % 2 else 0.5 * (m[n // 2 - 1] + m[n // 2])
    return {"min": m[0], "median": med, "max": m[-1], "empty": sum(1 for v in m if v == 0), "experts": n}


MXFP8_OPS_PER_CLK_SM = 16384  # dense MXFP8 tensor-core FLOPs per clock per SM (sm_100)


def clock_peak_tflops(sm_mhz: float, n_sm: int = 148) -> float:
    """Dense MXFP8 tensor-core peak at a given SM clock: 16384 FLOP per clock
    per SM x SMs x clock."""
    return MXFP8_OPS_PER_CLK_SM * n_sm * sm_mhz * 1e6 / 1e12


def phase_rates(cfg, fwd_ms: float, bwd_ms: float, peak: float, clk_peak) -> dict:
    """Layer forward / backward TFLOP/s and their fractions of the dense MXFP8
    peak (`peak`, the roofline denominator) and of the clock-based peak."""
    out = {}
    for name, fl, ms in (("fwd", cfg.fwd_flops(), fwd_ms), ("bwd", cfg.bwd_flops(), bwd_ms)):
        if not ms:
            continue
        tf = fl / (ms * 1e-3) / 1e12
        out[name] = {"ms": ms, "tflops": tf, "frac_of_peak": tf / peak,
                     "frac_of_clock_peak": (tf / clk_peak) if clk_peak else None}
    return out


def gemm_source_sha() -> str:
    h = hashlib.sha256()
    for rel in GEMM_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(cfg_name: str):
    """DRAM bytes per gate_up launch from the committed ncu summary, or None
    when the summary is missing, for another workload, or the kernel source
    changed since it was captured."""
    try:
        with open(PROFILE_SUMMARY) as fh:
            text = fh.read()
    except OSError:
        return None
    m_sha = re.search(r"source_sha256_16:\s*([0-9a-f]+)", text)
    m_b = re.search(r"traffic_bytes_per_launch_full:\s*([0-9.eE+]+)", text)
    m_w = re.search(r"workload:\s*(\S+)", text)
    if not (m_sha and m_b and m_w) or m_w.group(1) != cfg_name:
        return None
    if m_sha.group(1) != gemm_source_sha():
        return None
    return float(m_b.group(1))


def parse_clocks(csv_text: str, t0: float, t1: float):
    """nvidia-smi samples (timestamp, index, clocks.sm, clocks.max.sm,
    power, reasons...) -> summary over the samples inside [t0, t1] (the
    nearest ones if none fell inside)."""
    rows = []
    for line in csv_text.strip().splitlines():
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9 or not parts[2].replace(" MHz", "").isdigit():
            continue
        try:
            ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            continue
        rows.append((ts, int(parts[2].split()[0]), int(parts[3].split()[0]), parts[5:9]))
    if not rows:
        return None
    inside = [r for r in rows if t0 - 0.25 <= r[0] <= t1 + 0.25]
    if not inside:
        mid = 0.5 * (t0 + t1)
        inside = sorted(rows, key=lambda r: abs(r[0] - mid))[:3]
    mhz = sorted(r[1] for r in inside)
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3]) if v.lower() == "active"})
    return {"sm_mhz": mhz[len(mhz) // 2], "sm_max_mhz": max(r[2] for r in inside),
            "reasons": reasons, "samples": len(inside)}


class ClockSampler:
    """Background nvidia-smi sampler (200 ms) for one GPU index."""

    def __init__(self, index: int):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader",
                                          "-i", str(index), "-lms", "200"], stdout=self.file,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> str:
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        text = self.file.read()
        self.file.close()
        os.unlink(self.file.name)
        return text


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and --impl reference)
# ---------------------------------------------------------------------------

def oracle_sample(cfg, rows: int, seed: int, i_div: int = 1):
    """One bounded sample of the workload for the CPU oracle: `rows` routed
    rows of one expert and a 1/i_div slice of that expert's intermediate
    dimension (gate, up and down weights of those I/i_div channels; their
    weight quantisation in both directions included), forward + backward.
    Every element of the sample goes through the same arithmetic as in the
    full layer; the work scales linearly in rows and I.  Returns (seconds,
    algorithmic FLOPs of the sample, description)."""
    import numpy as np
    from oracle import moe as omoe
    rng = np.random.default_rng(seed)
    H, I = cfg.H, cfg.I // i_div
    x = rng.standard_normal((rows, H)).astype(np.float32).astype(np.float64)
    w1 = (rng.standard_normal((1, 2 * I, H)).astype(np.float32) / np.sqrt(H)).astype(np.float64)
    w2 = (rng.standard_normal((1, H, I)).astype(np.float32) / np.sqrt(I)).astype(np.float64)
    dy = rng.standard_normal((rows, H)).astype(np.float32).astype(np.float64)
    idx = np.zeros((rows, 1), np.int32)
    prob = rng.uniform(0.2, 0.8, (rows, 1)).astype(np.float32)
    t = time.perf_counter()
    f = omoe.forward(x, w1, w2, idx, prob)
    omoe.backward(f, x, w1, w2, prob, dy)
    dt = time.perf_counter() - t
    flops = 18.0 * rows * H * I
    desc = (f"{rows} routed rows of one expert of {cfg.name}, H={H}, a 1/{i_div} slice of I "
            f"({I} of {cfg.I} channels) with those weights; their MXFP8 quantisation in both "
            f"directions included; fwd+bwd; float64 numpy")
    return dt, flops, desc


def cpu_cores() -> int:
    """Threads the oracle runs on: the BLAS pool numpy's matrix products use
    (the bulk of its work; the rest is single-threaded numpy), else the
    host cores this process may use."""
    try:
        from threadpoolctl import threadpool_info
        blas = [p.get("num_threads", 0) for p in threadpool_info() if p.get("user_api") == "blas"]
        if blas and max(blas) > 0:
            return int(max(blas))
    except Exception:  # threadpoolctl missing or unable to inspect the BLAS
        pass
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run_reference(args):
    """--impl reference: the CPU oracle as it stands, timed on the host
    cores on bounded samples of the same workload.  Under torchrun only
    rank 0 runs it."""
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    cfg = get_config(args.config)
    rows, i_div = 64, 16
    for _ in range(args.warmup):
        oracle_sample(cfg, rows, args.seed, i_div)
    tot_t = tot_f = 0.0
    desc = ""
    for s in range(args.steps):
        dt, fl, desc = oracle_sample(cfg, rows, args.seed + s, i_div)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{cfg.name} expert layer fwd+bwd", "T": cfg.T, "H": cfg.H, "I": cfg.I,
                       "E": cfg.E, "k": cfg.k, "R": cfg.R,
                       "step": "weight quant (both directions) + permute + fwd + bwd",
                       "sample_rows_per_step": rows, "sample_i_fraction": f"1/{i_div}"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def make_device_inputs(torch, cfg, seed: int, dev):
    """Seeded synthetic inputs drawn on the device with the recipe of
    mxfp8_grouped_gemm_x32_b200.workloads (bf16 normals, N(0, 1/fan_in)
    weights, softmax/top-k routing renormalised)."""
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
    x = torch.randn(T, H, generator=g, device=dev).to(torch.bfloat16)
    w1 = (torch.randn(E, 2 * I, H, generator=g, device=dev) / H ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn(E, H, I, generator=g, device=dev) / I ** 0.5).to(torch.bfloat16)
    dy = torch.randn(T, H, generator=g, device=dev).to(torch.bfloat16)
    logits = torch.randn(T, E, generator=g, device=dev, dtype=torch.float64)
    if cfg.expert_bias_std:
        logits = logits + cfg.expert_bias_std * torch.randn(E, generator=g, device=dev, dtype=torch.float64)
    if cfg.router == "topk_softmax":
        top, idx = torch.topk(logits, k, dim=1)
        prob = torch.softmax(top, dim=1)
    else:
        p = torch.softmax(logits, dim=1)
        prob, idx = torch.topk(p, k, dim=1)
        prob = prob / prob.sum(dim=1, keepdim=True)
    return x, idx.to(torch.int32).contiguous(), prob.to(torch.float32).contiguous(), w1, w2, dy


class PhaseTimer:
    """CUDA events recorded on the launching stream between the phases of
    each step: weight quantisation | permutation + forward | backward."""

    def __init__(self, torch, n_steps: int):
        self.ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_steps)]
        self.i = 0

    def take(self):
        if self.i >= len(self.ev):
            return None
        e = self.ev[self.i]
        self.i += 1
        return e

    def phases(self):
        """Per-step (weight quant, fwd, bwd) in ms for the steps recorded."""
        return [(a.elapsed_time(b), b.elapsed_time(c), c.elapsed_time(d)) for a, b, c, d in self.ev[:self.i]]


def median(v):
    v = sorted(v)
    n = len(v)
    return v[n // 2] if n % 2 else 0.5 * (v[n // 2 - 1] + v[n // 2])


def make_step(layer, stream, x, idx, prob, w1, w2, dy):
    """One step of the layer; `rec` (four CUDA events) brackets its phases."""
    def step(rec=None):
        if rec:
            rec[0].record(stream)
        layer.quantize_weights(w1, w2)
        if rec:
            rec[1].record(stream)
        layer.permute(x, idx, prob)
        layer.forward()
        if rec:
            rec[2].record(stream)
        layer.backward(dy)
        if rec:
            rec[3].record(stream)
    return step


def measure_workload(torch, lib, name: str, seed: int, dev, steps: int, warmup: int, local: int, peaks) -> dict:
    """A further layer shape measured in the same run (1 GPU): `warmup`
    untimed steps, then `steps` steps, each preceded by a 256 MB write that
    flushes L2 (outside the timed phases).  Reports per-step medians of the
    layer forward, backward and weight quantisation, their TFLOP/s and
    fractions of the dense MXFP8 peak and of the clock-based peak, the
    per-kernel times and the rows-per-expert histogram."""
    from mxfp8_grouped_gemm_x32_b200.layer import GroupedMLP
    cfg = get_config(name)
    x, idx, prob, w1, w2, dy = make_device_inputs(torch, cfg, seed, dev)
    layer = GroupedMLP(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, device=dev)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)
    step = make_step(layer, stream, x, idx, prob, w1, w2, dy)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    st = layer.device_status()
    if st != 0:
        raise SystemExit(f"{name}: device status after warm-up: {lib.status_string(st)}")
    pt = PhaseTimer(torch, steps)
    sampler = ClockSampler(local)
    time.sleep(0.3)
    lib.moe_timing_enable(True)
    lib.moe_timing_read()
    t0 = time.time()
    for _ in range(steps):
        flush.fill_(1)
        step(pt.take())
    torch.cuda.synchronize()
    t1 = time.time()
    per_kernel = lib.moe_timing_read()
    lib.moe_timing_enable(False)
    time.sleep(0.3)
    clocks = parse_clocks(sampler.stop(), t0, t1)
    st = layer.device_status()
    if st != 0:
        raise SystemExit(f"{name}: device status after timing: {lib.status_string(st)}")
    ph = pt.phases()
    wq, fwd, bwd = (median([p[i] for p in ph]) for i in range(3))
    step_ms = median([sum(p) for p in ph])
    clk_peak = clock_peak_tflops(clocks["sm_mhz"]) if clocks else None
    flops = step_flops(cfg)
    out = {"config": {"T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "k": cfg.k, "R": cfg.R,
                      "router": cfg.router, "expert_bias_std": cfg.expert_bias_std},
           "steps": steps, "warmup": warmup, "timing": "median over steps; L2 flushed (256 MB write) before each step",
           "ms_per_step": step_ms, "tflops": flops / (step_ms * 1e-3) / 1e12,
           "frac_of_peak": flops / (step_ms * 1e-3) / 1e12 / peaks["mxfp8_sustained"],
           "weight_quant_ms": wq,
           "layer": phase_rates(cfg, fwd, bwd, peaks["mxfp8_sustained"], clk_peak),
           "peak_tflops": peaks["mxfp8_sustained"], "clock_peak_tflops": clk_peak,
           "rows_per_expert": split_histogram(layer.split_sizes.cpu().tolist()),
           "kernels": annotate_bandwidth({k: {"ms_per_step": v[0] / steps, "launches_per_step": v[1] / steps}
                                          for k, v in per_kernel.items()}, cfg, peaks["hbm_gbs"]),
           "clocks": clocks}
    del layer, flush
    torch.cuda.empty_cache()
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the product path has no CPU fallback)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    from mxfp8_grouped_gemm_x32_b200 import lib
    from mxfp8_grouped_gemm_x32_b200.layer import GroupedMLP

    cfg = get_config(args.config)
    x, idx, prob, w1, w2, dy = make_device_inputs(torch, cfg, args.seed + rank, dev)
    layer = GroupedMLP(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, device=dev)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    step = make_step(layer, stream, x, idx, prob, w1, w2, dy)
    for _ in range(args.warmup):
        step()
    st = layer.device_status()
    if st != 0:
        raise SystemExit(f"device status after warm-up: {lib.status_string(st)}")

    # ---- timed region: K steps, inputs resident in HBM --------------------
    pt = PhaseTimer(torch, args.steps)
    sampler = ClockSampler(local)
    time.sleep(0.3)
    lib.moe_timing_enable(True)
    lib.moe_timing_read()
    barrier()
    launches0 = lib.moe_launch_count()
    t_wall0 = time.time()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step(pt.take())
    e1.record(stream)
    barrier()
    t_wall1 = time.time()
    launches = lib.moe_launch_count() - launches0
    per_kernel = lib.moe_timing_read()
    lib.moe_timing_enable(False)
    time.sleep(0.3)
    clocks = parse_clocks(sampler.stop(), t_wall0, t_wall1)
    ms_max = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    flops = step_flops(cfg)
    value = world * flops / (ms_max * 1e-3) / 1e12
    ph = pt.phases()
    wq_ms, fwd_ms, bwd_ms = (sum(p[i] for p in ph) / len(ph) for i in range(3))

    # ---- end to end through the public API with host buffers --------------
    # Every step copies its own inputs (x, routing, dY) from pinned host memory
    # and reads its results (out, dX, dprob) back, as a training loop does: on a
    # copy stream, the inputs of step i+1 come in and the results of step i
    # leave while the next step computes (two buffer sets; results are
    # snapshotted on the device so the next step may overwrite the layer's).
    hin = tuple(t.cpu().pin_memory() for t in (x, idx, prob, dy))
    h2d = sum(t.numel() * t.element_size() for t in hin)
    outs = (layer.out, layer.dX, layer.dprob)
    d2h = sum(t.numel() * t.element_size() for t in outs)
    din = [tuple(torch.empty_like(t) for t in (x, idx, prob, dy)) for _ in range(2)]
    dsnap = [tuple(torch.empty_like(t) for t in outs) for _ in range(2)]
    hout = [tuple(torch.empty_like(t, device="cpu").pin_memory() for t in outs) for _ in range(2)]
    copy = torch.cuda.Stream(device=dev)
    ev_in, ev_free, ev_out, ev_read = ([torch.cuda.Event() for _ in range(2)] for _ in range(4))

    def e2e_h2d(b):
        with torch.cuda.stream(copy):
            copy.wait_event(ev_free[b])            # the step that last read buffer b is done
            for d, h in zip(din[b], hin):
                d.copy_(h, non_blocking=True)
            ev_in[b].record(copy)

    def e2e_compute(b):
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_read[b])              # snapshot b has been read back
        xb, ib, pb, dyb = din[b]
        layer.step(xb, ib, pb, w1, w2, dyb)
        ev_free[b].record(stream)
        for d, t in zip(dsnap[b], outs):
            d.copy_(t, non_blocking=True)
        ev_out[b].record(stream)

    def e2e_d2h(b):
        with torch.cuda.stream(copy):
            copy.wait_event(ev_out[b])
            for h, d in zip(hout[b], dsnap[b]):
                h.copy_(d, non_blocking=True)
            ev_read[b].record(copy)

    def e2e_run(n):
        e2e_h2d(0)
        for i in range(n):
            if i + 1 < n:
                e2e_h2d((i + 1) % 2)
            e2e_compute(i % 2)
            e2e_d2h(i % 2)
        stream.wait_event(ev_read[(n - 1) % 2])    # the last results are on the host

    e2e_run(2)
    torch.cuda.synchronize()
    barrier()
    e0.record(stream)
    e2e_run(args.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    value_e2e = world * flops / (ms_e2e * 1e-3) / 1e12
    # router (moe_router_topk): reported beside the step, which starts from
    # top-k routing; fp32 logits of the workload's shape
    glog = torch.Generator(device=dev)
    glog.manual_seed(args.seed + 7)
    logits = torch.randn(cfg.T, cfg.E, generator=glog, device=dev)
    for _ in range(3):
        layer.route(logits)
    e0.record(stream)
    for _ in range(20):
        layer.route(logits)
    e1.record(stream)
    torch.cuda.synchronize()
    router_ms = e0.elapsed_time(e1) / 20
    st = layer.device_status()
    if st != 0:
        raise SystemExit(f"device status after timing: {lib.status_string(st)}")
    split_host = layer.split_sizes.cpu().tolist()
    # forward-only layer (inference): weights quantised once, then permutation +
    # forward per call, no saved activation and no quantisation along tokens
    inf = GroupedMLP(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, device=dev, backward=False)
    inf.quantize_weights(w1, w2)
    for _ in range(3):
        inf.permute(x, idx, prob)
        inf.forward()
    e0.record(stream)
    for _ in range(10):
        inf.permute(x, idx, prob)
        inf.forward()
    e1.record(stream)
    torch.cuda.synchronize()
    ms_inf = max_over_ranks(e0.elapsed_time(e1) / 10, world, dev)
    del inf
    # the BF16 recipe's forward (bf16 operands, no MXFP8): routing + forward
    for _ in range(3):
        layer.permute_index(idx, prob)
        layer.forward_bf16(x, w1, w2)
    e0.record(stream)
    for _ in range(10):
        layer.permute_index(idx, prob)
        layer.forward_bf16(x, w1, w2)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_bf16 = max_over_ranks(e0.elapsed_time(e1) / 10, world, dev)
    st = layer.device_status()
    if st != 0:
        raise SystemExit(f"device status after the BF16 forward: {lib.status_string(st)}")
    # the BF16 recipe's training step: routing + forward (saving A) + backward
    for _ in range(3):
        layer.permute_index(idx, prob)
        layer.forward_bf16(x, w1, w2)
        layer.backward_bf16(dy, x, w1, w2)
    e0.record(stream)
    for _ in range(10):
        layer.permute_index(idx, prob)
        layer.forward_bf16(x, w1, w2)
        layer.backward_bf16(dy, x, w1, w2)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_bf16_step = max_over_ranks(e0.elapsed_time(e1) / 10, world, dev)
    st = layer.device_status()
    if st != 0:
        raise SystemExit(f"device status after the BF16 backward: {lib.status_string(st)}")
    # the per-tensor FP8 recipe's forward (one factor per tensor, quantised
    # from the bf16 weights and x every call): routing + forward
    for _ in range(3):
        layer.permute_index(idx, prob)
        layer.forward_fp8_tensor(x, w1, w2)
    e0.record(stream)
    for _ in range(10):
        layer.permute_index(idx, prob)
        layer.forward_fp8_tensor(x, w1, w2)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_f8t = max_over_ranks(e0.elapsed_time(e1) / 10, world, dev)
    st = layer.device_status()
    if st != 0:
        raise SystemExit(f"device status after the per-tensor FP8 forward: {lib.status_string(st)}")
    # the per-tensor FP8 recipe's training step: routing + forward (saving A)
    # + backward
    for _ in range(3):
        layer.permute_index(idx, prob)
        layer.forward_fp8_tensor(x, w1, w2)
        layer.backward_fp8_tensor(dy, x, w1, w2)
    e0.record(stream)
    for _ in range(10):
        layer.permute_index(idx, prob)
        layer.forward_fp8_tensor(x, w1, w2)
        layer.backward_fp8_tensor(dy, x, w1, w2)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_f8t_step = max_over_ranks(e0.elapsed_time(e1) / 10, world, dev)
    st = layer.device_status()
    if st != 0:
        raise SystemExit(f"device status after the per-tensor FP8 backward: {lib.status_string(st)}")

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks = load_peaks()
    peak = peaks["mxfp8_sustained"]
    clk_peak = clock_peak_tflops(clocks["sm_mhz"]) if clocks else None
    kernels = annotate_bandwidth({k: {"ms_per_step": v[0] / args.steps, "launches_per_step": v[1] / args.steps}
                                  for k, v in per_kernel.items()}, cfg, peaks["hbm_gbs"])
    g1 = per_kernel.get("gemm_gate_up_swiglu")
    roofline = None
    if g1 and g1[1]:
        t_launch = g1[0] / g1[1] * 1e-3
        achieved = gate_up_flops(cfg) / t_launch / 1e12
        roofline = {"bound": "tensor", "kernel": "gemm_gate_up_swiglu", "achieved": achieved,
                    "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                    "traffic": profiled_traffic(cfg.name),
                    "peak_source": f"{peaks['source']} bf16 sustained x {MXFP8_OVER_BF16} (nominal MXFP8/BF16)",
                    "frac_of_burst": achieved / peaks["mxfp8_burst"],
                    "frac_of_clock_peak": achieved / clk_peak if clk_peak else None}
    layer_rates = phase_rates(cfg, fwd_ms, bwd_ms, peak, clk_peak)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "mxfp8 (e4m3 x e4m3, e8m0 block scales, fp32 accumulate)",
        "data": "synthetic (seeded, drawn on device; bf16 N(0,1) tokens, N(0,1/fan_in) weights, "
                "softmax top-k routing)",
        "config": {"workload": f"{cfg.name} expert layer fwd+bwd", "T": cfg.T, "H": cfg.H, "I": cfg.I,
                   "E": cfg.E, "k": cfg.k, "R": cfg.R, "parallelism": f"replicas x{world} (data-parallel tokens)",
                   "l2": l2_note(cfg),
                   "step": "weight quant (both directions) + permute + fwd + bwd",
                   "flops_per_step": flops},
        "frac_of_mxfp8_peak": value / world / peak,
        "clock_peak_tflops": clk_peak,
        "frac_of_clock_peak": value / world / clk_peak if clk_peak else None,
        # layer forward = permutation + forward; layer backward = the backward
        # call; CUDA events between the phases of every timed step (means)
        "layer": layer_rates,
        "fwd_tflops": layer_rates.get("fwd", {}).get("tflops"),
        "bwd_tflops": layer_rates.get("bwd", {}).get("tflops"),
        "weight_quant_ms": wq_ms,
        # the step without the weight quantisation: a gradient-accumulation
        # micro-step, where the MX weights of the optimizer step are reused
        "excl_weight_quant": {"value": world * flops / ((fwd_ms + bwd_ms) * 1e-3) / 1e12, "unit": "TFLOP/s",
                              "ms_per_step": fwd_ms + bwd_ms},
        "kernels": kernels,
        "rows_per_expert": split_histogram(split_host),
        "inference_fwd": {"value": world * cfg.fwd_flops() / (ms_inf * 1e-3) / 1e12, "unit": "TFLOP/s",
                          "ms_per_call": ms_inf,
                          "what": "forward-only layer: permutation + forward per call, MX weights reused"},
        "bf16_fwd": {"value": world * cfg.fwd_flops() / (ms_bf16 * 1e-3) / 1e12, "unit": "TFLOP/s",
                     "ms_per_call": ms_bf16, "peak_bf16_tflops": peaks["bf16_sustained"],
                     "frac_of_bf16_peak": cfg.fwd_flops() / (ms_bf16 * 1e-3) / 1e12 / peaks["bf16_sustained"],
                     "what": "BF16 recipe layer forward (moe_permute without x + moe_grouped_mlp_fwd_bf16): "
                             "bf16 operands, no MXFP8"},
        "bf16_step": {"value": world * flops / (ms_bf16_step * 1e-3) / 1e12, "unit": "TFLOP/s",
                      "ms_per_call": ms_bf16_step, "bwd_ms": ms_bf16_step - ms_bf16,
                      "bwd_tflops": cfg.bwd_flops() / ((ms_bf16_step - ms_bf16) * 1e-3) / 1e12,
                      "peak_bf16_tflops": peaks["bf16_sustained"],
                      "frac_of_bf16_peak": flops / (ms_bf16_step * 1e-3) / 1e12 / peaks["bf16_sustained"],
                      "what": "BF16 recipe layer step: moe_permute without x + moe_grouped_mlp_fwd_bf16 (saving A) "
                              "+ moe_grouped_mlp_bwd_bf16 (weights transposed in the call); bwd_ms = step - "
                              "bf16_fwd"},
        "fp8_tensor_fwd": {"value": world * cfg.fwd_flops() / (ms_f8t * 1e-3) / 1e12, "unit": "TFLOP/s",
                           "ms_per_call": ms_f8t,
                           "what": "per-tensor FP8 recipe layer forward (moe_permute without x + "
                                   "moe_grouped_mlp_fwd_fp8_tensor): factors from the current |max| of x, of every "
                                   "expert's weights and of h, weights quantised in the call"},
        "fp8_tensor_step": {"value": world * flops / (ms_f8t_step * 1e-3) / 1e12, "unit": "TFLOP/s",
                            "ms_per_call": ms_f8t_step, "bwd_ms": ms_f8t_step - ms_f8t,
                            "bwd_tflops": cfg.bwd_flops() / ((ms_f8t_step - ms_f8t) * 1e-3) / 1e12,
                            "what": "per-tensor FP8 recipe layer step: moe_permute without x + "
                                    "moe_grouped_mlp_fwd_fp8_tensor (saving A) + moe_grouped_mlp_bwd_fp8_tensor "
                                    "(dY, da, h factored in the call, weights transposed and coded in the call); "
                                    "bwd_ms = step - fp8_tensor_fwd"},
        "router": {"ms_per_call": router_ms, "in_step": False,
                   "what": "moe_router_topk on fp32 logits [T, E] (softmax, top-k, renormalise)"},
        "roofline": roofline,
        "clocks": clocks,
        "e2e": {"value": value_e2e, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": ms_e2e,
                "pipeline": "copy stream: inputs of step i+1 in, results of step i out, while step i+1 computes"},
        "gpu_launches": launches,
    }
    # attainable layer forward for this routing (per-expert max of compute and
    # bytes) at the roofline peak
    att = attainable_fwd(cfg, split_host, peak, peaks["hbm_gbs"], layer.rows_cap)
    att["measured_ms"] = fwd_ms
    att["frac"] = att["ms"] / fwd_ms
    line["attainable_fwd"] = att
    del layer, x, idx, prob, w1, w2, dy, din, dsnap
    torch.cuda.empty_cache()
    side = [n for n in args.workloads.split(",") if n and n not in ("none", cfg.name)]
    if world == 1 and side:
        # the other layer shapes, measured in the same run on the same GPU
        line["workloads"] = {}
        for name in side:
            line["workloads"][name] = measure_workload(torch, lib, name, args.seed, dev, max(args.steps, 50),
                                                       max(args.warmup, 10), local, peaks)
    if not args.no_library_probe:
        probe = mxfp8_library_probe(torch, dev)
        line["mxfp8_library_probe"] = probe
        if "sustained_tflops" in probe:
            lib_s = probe["sustained_tflops"]
            probe["frac"] = {"step": value / world / lib_s,
                             "layer_fwd": (line["fwd_tflops"] or 0.0) / lib_s,
                             "layer_bwd": (line["bwd_tflops"] or 0.0) / lib_s}
            probe["note"] = "context only: a library's achieved rate, not the peak the targets use"
    if world == 1 and not args.no_cpu_baseline:
        dt, fl, desc = oracle_sample(cfg, 256, args.seed, 4)
        line["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(),
                                "kind": "oracle", "sample": desc, "seconds": dt}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
