"""The benchmark's multi-rank plumbing on CPU: two gloo ranks, as torchrun
would launch them, agree on the slowest rank's time, pass the barrier and
report whole-job throughput; under the reference arm only rank 0 works."""
import contextlib
import io
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, results):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world)})
    ranks = bench.Ranks("gloo", timeout_s=60)
    assert (ranks.rank, ranks.world) == (rank, world)
    ranks.barrier()
    slowest = ranks.max(10.0 + rank)  # rank r took 10 + r ms
    results[rank] = (slowest, bench.aggregate_rate(1000, ranks.world, slowest))
    ranks.close()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world, port = 2, _free_port()
    results = mp.Manager().dict()
    mp.start_processes(_rank_main, args=(world, port, results), nprocs=world, start_method="spawn", join=True)
    assert sorted(results.keys()) == [0, 1]
    for r in range(world):
        slowest, rate = results[r]
        assert slowest == pytest.approx(11.0)
        # 2 replicas x 1000 tokens in the slowest rank's 11 ms
        assert rate == pytest.approx(2000 / 11e-3)


def test_single_process_needs_no_process_group():
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        os.environ.pop(k, None)
    ranks = bench.Ranks("gloo")
    assert ranks.world == 1 and ranks.dist is None
    assert ranks.max(3.5) == 3.5
    ranks.barrier()
    ranks.close()


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
                                      "--warmup", "1"])
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.main()
    assert out.getvalue() == ""


def test_fp8_reference_arm_times_the_fp8_oracle(monkeypatch):
    import json
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--fp8-quant", "--steps", "2",
                                      "--warmup", "1", "--cpu-sample", "16"])
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.main()
    line = json.loads(out.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.FP8_METRIC and line["unit"] == "GB/s"
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["config"]["workload"].startswith("16b_prefill")


def test_reference_arm_times_the_oracle_on_one_thread(monkeypatch):
    import json
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--config", "tiny", "--steps", "2",
                                      "--warmup", "1"])
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.main()
    line = json.loads(out.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["cores"] == 1 and line["cpu_baseline"]["host_cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_peak_follows_the_length_and_clock_of_the_timed_region():
    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1667.0, "bf16_tflops_sustained": 1397.0}
    at_max = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    capped = {"sm_mhz": 1400.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.choose_peak(peaks, 0.04, at_max) == (1667.0, "bf16_tflops")
    assert bench.choose_peak(peaks, 0.04, None) == (1667.0, "bf16_tflops")
    assert bench.choose_peak(peaks, 2.5, at_max) == (1397.0, "bf16_tflops_sustained")
    assert bench.choose_peak(peaks, 0.04, capped) == (1397.0, "bf16_tflops_sustained")


def test_roofline_of_the_dominant_kernel_from_its_own_numbers():
    import workloads as W
    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1667.0, "bf16_tflops_sustained": 1397.0}
    clk = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    shape = W.CONFIGS["16b_prefill"]
    r = {"ms_total": 41.0, "ms_step": 2.05, "clocks": clk, "dominant_ms": 1.2252, "counts": [1536] * 64,
         "kernel_ms": {"gate_up": 1.2252, "down": 0.56}}
    roof, peak, _ = bench.roofline_of(shape, r, peaks, "measured")
    flop = 4.0 * 16384 * 2048 * (6 * 1408 + 2 * 1408)
    assert roof["bound"] == "tensor" and roof["flop_per_launch"] == flop
    assert roof["achieved"] == pytest.approx(flop / 1.2252e-3 / 1e12)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 1667.0) and peak == 1667.0
    # a decode batch: both expert GEMMs are one launch (timed as gate_up), over all three projections
    decode = W.CONFIGS["16b_decode"]
    counts = [6] * 30 + [0] * 34                  # 30 of the 64 experts touched
    r = dict(r, ms_total=20.0, ms_step=0.13, dominant_ms=0.11, counts=counts,
             kernel_ms={"gate_up": 0.11, "down": 0.0})
    roof, _, _ = bench.roofline_of(decode, r, peaks, "measured")
    wbytes = 3 * 2 * 2048 * (30 * 1408 + 2 * 1408)
    assert roof["bound"] == "hbm" and roof["weight_bytes_per_launch"] == wbytes
    assert roof["flop_per_launch"] == 6.0 * 32 * 2048 * (6 * 1408 + 2 * 1408)
    assert roof["achieved"] == pytest.approx(wbytes / 0.11e-3 / 1e9)
    assert "decode_ffn_kernel" in roof["kernel"]
    f = bench.hbm_fractions(decode, r, peaks)
    assert f["ffn_gbs"] == pytest.approx(wbytes / 0.11e-3 / 1e9) and "down_gbs" not in f
    assert f["layer_frac"] == pytest.approx(wbytes / 0.13e-3 / 1e9 / 6500.0)
    # the FP8 layer's decode batches too run both GEMMs in one launch, over 1-byte weights and their scales
    f8 = bench.hbm_fractions(decode, dict(r, kernel_ms={"gate_up": 0.07, "down": 0.0}), peaks, fp8=True)
    b8 = 3 * (1.0 + 1.0 / (128 * 128)) * 2048 * (30 * 1408 + 2 * 1408)
    assert f8["ffn_gbs"] == pytest.approx(b8 / 0.07e-3 / 1e9) and "down_gbs" not in f8
    roof8, _, _ = bench.roofline_of(decode, dict(r, dominant_ms=0.07), peaks, "measured", fp8=True)
    assert roof8["bound"] == "hbm" and "decode_ffn8_kernel" in roof8["kernel"]
    # a prefill batch keeps separate GEMM launches
    f16 = bench.hbm_fractions(W.CONFIGS["v3"], dict(r, kernel_ms={"gate_up": 3.6, "down": 2.0},
                                                      counts=[128] * 256), peaks)
    assert f16["down_gbs"] is not None and "ffn_gbs" not in f16
