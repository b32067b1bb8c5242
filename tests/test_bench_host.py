"""Host logic of bench.py (no GPU): FLOP accounting, peaks, provenance of
the profiled traffic, nvidia-smi clock parsing, and the multi-process path
-- the max-over-ranks step time under a 2-rank gloo process group on CPU,
and the reference arm's rank handling."""
import json
import os
import socket

import pytest

import bench
from mxfp8_grouped_gemm_x32_b200.workloads import get_config


def test_step_flops_mixtral():
    cfg = get_config("mixtral_8x7b")
    R, H, I = 16384, 4096, 14336
    assert bench.step_flops(cfg) == 18.0 * R * H * I
    assert bench.gate_up_flops(cfg) == 2.0 * R * H * 2 * I


def test_load_peaks(tmp_path):
    p = tmp_path / "peaks.json"
    p.write_text(json.dumps({"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}))
    pk = bench.load_peaks(str(p))
    assert pk["source"] == "measured" and pk["mxfp8_burst"] == 3200.0 and pk["mxfp8_sustained"] == 2800.0
    fb = bench.load_peaks(str(tmp_path / "missing.json"))
    assert fb["source"] == "fallback" and fb["mxfp8_burst"] == 2 * 1590.0


def test_profiled_traffic_tracks_kernel_source(tmp_path, monkeypatch):
    sha = bench.gemm_source_sha()
    f = tmp_path / "summary.md"
    f.write_text(f"workload: mixtral_8x7b\nsource_sha256_16: {sha}\ntraffic_bytes_per_launch_full: 2.0e9\n")
    monkeypatch.setattr(bench, "PROFILE_SUMMARY", str(f))
    assert bench.profiled_traffic("mixtral_8x7b") == 2.0e9
    assert bench.profiled_traffic("gpt_oss_20b") is None
    f.write_text("workload: mixtral_8x7b\nsource_sha256_16: 0000000000000000\ntraffic_bytes_per_launch_full: 2e9\n")
    assert bench.profiled_traffic("mixtral_8x7b") is None


def test_parse_clocks():
    csv = ("2026/12/02 16:00:00.000, 0, 1900 MHz, 1965 MHz, 900.00 W, Not Active, Not Active, Not Active, Active\n"
           "2026/12/02 16:00:00.200, 0, 1950 MHz, 1965 MHz, 950.00 W, Not Active, Not Active, Not Active, Not Active\n"
           "2026/12/02 16:00:00.400, 0, 1800 MHz, 1965 MHz, 990.00 W, Not Active, Not Active, Not Active, Active\n"
           "2026/12/02 16:00:05.000, 0, 300 MHz, 1965 MHz, 100.00 W, Not Active, Not Active, Not Active, Not Active\n")
    import datetime
    t0 = datetime.datetime(2026, 12, 2, 16, 0, 0).timestamp()
    c = bench.parse_clocks(csv, t0, t0 + 0.4)
    assert c["sm_mhz"] == 1900 and c["sm_max_mhz"] == 1965 and c["samples"] == 3
    assert c["reasons"] == ["sw_power_cap"]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        v = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        with open(os.path.join(out_dir, f"r{rank}"), "w") as fh:
            fh.write(repr(v))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_processes(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    vals = [float((tmp_path / f"r{r}").read_text()) for r in range(2)]
    assert vals == [15.0, 15.0]


def test_reference_arm_non_zero_rank_exits_without_output(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0"]) == 0
    assert capsys.readouterr().out == ""


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_attainable_fwd_limits():
    """The attainable forward is the sum over experts of the larger of the
    compute and byte times: with no bandwidth limit it is FLOPs / P plus the
    permutation and combine bytes; an expert with no rows still streams its
    weights; more rows never make it smaller."""
    cfg = get_config("tiny")                          # H256 I512 E4 k2, T512
    H, I, T, k = cfg.H, cfg.I, cfg.T, cfg.k
    split = [256, 256, 256, 256]
    big_bw = bench.attainable_fwd(cfg, split, 1000.0, 1e12, 1536)["ms"]
    flops = sum(6.0 * m * H * I for m in split)
    pc_bytes = T * H * 2 + T * k * H * (1 + 1 / 32) + T * k * H * 3 + T * H * 2
    assert big_bw == pytest.approx((flops / 1e15 + pc_bytes / 1e21) * 1e3, rel=1e-12)  # GEMM bytes take no time
    empty = bench.attainable_fwd(cfg, [0, 0, 0, 1024], 1e9, 1000.0, 1536)["ms"]
    w_bytes = 3 * (1 + 1 / 32) * H * I                               # MX W_gate_up + W_down of one expert
    assert empty >= 3 * w_bytes / 1e12 * 1e3                         # the three idle experts still read weights
    a = bench.attainable_fwd(cfg, [100, 200, 300, 424], 2000.0, 6000.0, 1536)["ms"]
    b = bench.attainable_fwd(cfg, [200, 200, 300, 424], 2000.0, 6000.0, 1536)["ms"]
    assert b >= a


def test_bandwidth_annotation():
    """Bandwidth kernels get algorithmic bytes, GB/s and the HBM fraction;
    other kernels are left as they are."""
    cfg = get_config("mixtral_8x7b")                  # T8192 H4096 I14336 E8 k2
    b = bench.bandwidth_bytes(cfg)
    mx = 1 + 1 / 32
    assert b["quant_weights"] == pytest.approx(3 * 8 * 4096 * 14336 * (2 + 2 * mx))   # 5.71 GB
    assert b["permute_quant"] == pytest.approx(8192 * 4096 * 2 + 16384 * 4096 * mx)
    assert b["dy_quant"] == pytest.approx(8192 * 4096 * 2 + 2 * 16384 * 4096 * mx)
    assert b["combine"] == pytest.approx(16384 * 4096 * 3 + 8192 * 4096 * 2)
    k = bench.annotate_bandwidth({"combine": {"ms_per_step": 0.05}, "gemm_down": {"ms_per_step": 0.9}}, cfg, 6650.0)
    assert k["combine"]["gbs"] == pytest.approx(b["combine"] / 0.05e-3 / 1e9)
    assert k["combine"]["frac_of_hbm"] == pytest.approx(k["combine"]["gbs"] / 6650.0)
    assert "gbs" not in k["gemm_down"]


def test_l2_note_states_the_weight_bytes():
    assert bench.l2_note(get_config("mixtral_8x7b")).startswith("inputs larger than L2 (bf16 weights 2.82 GB")
    assert "1.21 GB" in bench.l2_note(get_config("qwen3_30b_ragged"))
    assert "1.59 GB" in bench.l2_note(get_config("gpt_oss_20b"))
    assert bench.l2_note(get_config("tiny")).startswith("inputs smaller than L2")


def test_cpu_cores_reports_the_blas_threads():
    import numpy  # noqa: F401  (loads the BLAS the oracle uses)
    from threadpoolctl import threadpool_info, threadpool_limits
    if not any(p.get("user_api") == "blas" for p in threadpool_info()):
        pytest.skip("no BLAS pool visible")
    with threadpool_limits(limits=1, user_api="blas"):
        assert bench.cpu_cores() == 1
    assert bench.cpu_cores() >= 1


def test_split_histogram_and_peaks():
    h = bench.split_histogram([0, 5, 3, 0, 100, 7])
    assert h == {"min": 0, "median": 4.0, "max": 100, "empty": 2, "experts": 6}
    assert bench.split_histogram([4, 1, 9])["median"] == 4
    # 16384 FLOP per clock per SM x 148 SMs at 1.965 GHz
    assert abs(bench.clock_peak_tflops(1965) - 16384 * 148 * 1.965e9 / 1e12) < 1e-9
    cfg = get_config("qwen3_30b_ragged")
    r = bench.phase_rates(cfg, 1.0, 2.0, 2800.0, 4000.0)
    assert abs(r["fwd"]["tflops"] - cfg.fwd_flops() / 1e-3 / 1e12) < 1e-6
    assert abs(r["bwd"]["frac_of_peak"] - cfg.bwd_flops() / 2e-3 / 1e12 / 2800.0) < 1e-12
    assert abs(r["fwd"]["frac_of_clock_peak"] - r["fwd"]["tflops"] / 4000.0) < 1e-12
    assert bench.phase_rates(cfg, 1.0, 0.0, 2800.0, None)["fwd"]["frac_of_clock_peak"] is None
