#!/usr/bin/env python
"""Benchmark of the DeepSeekMoE layer forward on B200.

One step = one full layer forward (router + top-K, permutation, routed
gate/up + SwiGLU, routed down + gate scale, shared experts, final sum) over
one batch of T synthetic tokens already resident in HBM.  The default
workload is the DeepSeekMoE-16B-shaped prefill layer (T=16384, d=2048,
64 routed experts of 1408, top-6, 2 shared experts of 1408).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0.  ``--impl reference`` times the CPU oracle
(the plain float64 restatement of the layer) on a bounded sample of the same
workload.  Under torchrun every rank runs an independent replica (the layer
has no data-path exchange on one GPU; replicas only), timed on the device and
reduced as the max over ranks.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "MoE layer fwd tokens/s; activated-expert TFLOP/s as % of B200 bf16 peak"
UNIT = "tokens/s"
L2_BYTES = 126 * 2**20
PEAK_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DOMINANT = "gate_up"
# batches of at most this many tokens run both expert GEMMs in one launch (the decode FFN), timed as gate_up
DECODE_MAX_T = 64
# committed ncu summaries of the dominant kernel (the gate/up GEMM of the path the workload runs), per
# (workload, fp8): the summary file and the sources whose hash it records; DRAM bytes per token
# (prefill) or per launch
_CSRC = "fine_grained_shared_b200/csrc/"
KERNEL_SOURCES = [_CSRC + "gateup_gemm.cuh", _CSRC + "sm100.cuh"]
PROFILE_SUMMARIES = {
    ("16b_prefill", False): (os.path.join(ROOT, "profiles", "gate_up_16b_prefill.txt"), KERNEL_SOURCES),
    ("16b_decode", False): (os.path.join(ROOT, "profiles", "decode_ffn_16b_decode.txt"),
                            [_CSRC + "decode_ffn.cuh", _CSRC + "sm100.cuh"]),
    ("16b_prefill", True): (os.path.join(ROOT, "profiles", "fp8_gemms_16b_prefill.txt"),
                            [_CSRC + "fp8_gemm.cuh", _CSRC + "fp8_util.cuh", _CSRC + "sm100.cuh"]),
}
FP8_PROFILES = {"16b_prefill": os.path.join(ROOT, "profiles", "fp8_quant_rows_16b_prefill.txt")}
FP8_SOURCES = ["fine_grained_shared_b200/csrc/fp8_quant.cu"]


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=400)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--config", default="16b_prefill", choices=sorted(W.CONFIGS))
    p.add_argument("--cpu-sample", type=int, default=256, help="rows of the FP8 oracle's CPU-baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-per-config", action="store_true",
                   help="measure only the --config workload (by default the 2B, 16B decode and V3 layers follow)")
    p.add_argument("--fp8", action="store_true",
                   help="the layer with FP8 expert GEMMs (moe_forward_fp8) on the --config workload alone")
    p.add_argument("--fp8-quant", action="store_true",
                   help="time the FP8 1x128 quantization of one forward's permuted activations instead")
    p.add_argument("--training-step", action="store_true",
                   help="time only the layer's training step (forward + backward) on the --config workload")
    p.add_argument("--ep-emulate", type=int, default=0, metavar="G",
                   help="the expert-parallel layer with G ranks emulated on this GPU (each rank T / G tokens "
                        "and mN / G experts), against the single-GPU layer on the same tokens")
    return p.parse_args()


def workload_config(shape: W.LayerShape, parallelism: str) -> dict:
    return {"workload": f"deepseekmoe_layer_{shape.name}", "T": shape.T, "d_model": shape.d,
            "n_routed": shape.N, "d_ff": shape.I, "top_k": shape.K, "n_shared": shape.Ks,
            "d_ff_shared": shape.Is, "gate": shape.gate, "bias": shape.bias,
            "global_batch": shape.T, "parallelism": parallelism,
            "l2": l2_note(shape)}


def l2_note(shape: W.LayerShape) -> str:
    gb = expert_weight_gb(shape)
    if gb * 1e9 > L2_BYTES:
        return (f"no flush: the expert weights a step reads (up to {gb:.2f} GB, the touched experts') "
                f"exceed the 126 MB L2")
    return f"no flush: the layer's {gb * 1e3:.1f} MB of weights fit in the 126 MB L2, so steps run L2-warm"


def expert_weight_gb(shape: W.LayerShape) -> float:
    return 3.0 * 2 * shape.d * (shape.N * shape.I + shape.Ks * shape.Is) / 1e9


def layer_flop(shape: W.LayerShape) -> float:
    return shape.routed_flop + shape.shared_flop + shape.router_flop


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return PEAK_FALLBACK, "fallback"


def kernel_source_hash(sources=KERNEL_SOURCES) -> str:
    h = hashlib.sha256()
    for p in sources:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(shape: W.LayerShape, path=None, sources=KERNEL_SOURCES, fp8: bool = False):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary of this workload, if it was taken on the current kernel source; else None."""
    if path is None:
        path, sources = PROFILE_SUMMARIES.get((shape.name, fp8), (None, sources))
    if path is None or not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                vals.setdefault(k.strip(), v.strip())  # the first kernel listed is the dominant one
    if vals.get("source_sha256_16") != kernel_source_hash(sources):
        return None
    try:
        if "traffic_bytes_per_token" in vals:
            return float(vals["traffic_bytes_per_token"]) * shape.T
        return float(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------------------
# clocks sampled with nvidia-smi during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            gpu = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 8]
        if not rows:
            return None
        sm = [float(r[0]) for r in rows]
        mx = float(rows[0][1])
        busy = [s for s in sm if s > 0.5 * mx] or sm
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for i, n in enumerate(names):
                if r[4 + i].strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(rows), "power_w_max": max(float(r[2]) for r in rows)}


# ---------------------------------------------------------------------------
# inputs
# ---------------------------------------------------------------------------

def host_inputs(shape: W.LayerShape):
    return W.layer_inputs(shape, with_experts=True)


def to_device(host: dict, dev) -> dict:
    return {k: (v.to(dev) if v is not None else None) for k, v in host.items()}


# ---------------------------------------------------------------------------
# CPU oracle timing (the baseline arm)
# ---------------------------------------------------------------------------

def host_cpu():
    """(logical cores, CPU model) of the host."""
    model = ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return os.cpu_count() or 1, model


def oracle_tokens_per_s(shape: W.LayerShape, host: dict, n_tokens: int, repeats: int = 1, fp8: bool = False):
    """The CPU oracle, as it stands, on ``n_tokens`` seeded tokens of the batch, on ONE thread (numpy's
    BLAS limited to one thread for the call): the plain single-threaded baseline.  fp8: the FP8 layer's
    oracle (expert operands quantized as the FP8 path quantizes them)."""
    import oracle as O
    import oracle.fp8 as F8
    from threadpoolctl import threadpool_limits
    rows = W.sample_tokens(shape, n_tokens)
    ex = (host["w_gate"], host["w_up"], host["w_down"])
    sh = (host["ws_gate"], host["ws_up"], host["ws_down"]) if shape.Ks else None
    fwd = F8.moe_forward_fp8 if fp8 else O.moe_forward
    times = []
    with threadpool_limits(limits=1):
        for _ in range(repeats):
            t0 = time.perf_counter()
            fwd(host["x"], host["router"], shape.K, ex, sh, gate_kind=shape.gate,
                logit_bias=host["logit_bias"], select_bias=host["select_bias"], rows=rows)
            times.append(time.perf_counter() - t0)
    return rows.size, times, 1


def cpu_baseline(shape: W.LayerShape, host: dict, seconds: float = 15.0, max_tokens: int = 4096,
                 fp8: bool = False):
    """The oracle on a bounded sample sized to about ``seconds`` of one core's work (calibrated on 64
    tokens, which already pay the per-expert weight conversions)."""
    n_cal, t_cal, _ = oracle_tokens_per_s(shape, host, 64, fp8=fp8)
    n = int(max(8, min(shape.T, max_tokens, seconds * n_cal / max(t_cal[0], 1e-6))))
    n, times, threads = oracle_tokens_per_s(shape, host, n, fp8=fp8)
    cores, model = host_cpu()
    return {"value": n / times[0], "unit": UNIT, "cores": threads, "kind": "oracle",
            "host_cores": cores, "cpu_model": model,
            "sample": f"{n} seeded tokens of the T={shape.T} batch (routing, routed and shared experts, final "
                      f"sum; {'the FP8 layer, ' if fp8 else ''}float64 numpy on one thread), {times[0]:.1f} s"}


def run_reference(args):
    shape = W.CONFIGS[args.config]
    host = host_inputs(shape)
    # size each step's sample so that warmup + steps finish in about three minutes
    n_cal, t_cal, threads = oracle_tokens_per_s(shape, host, 4)
    cores, model = host_cpu()
    per_token = t_cal[0] / n_cal
    budget = 180.0 / max(1, args.steps + args.warmup)
    n = int(max(1, min(shape.T, budget / per_token)))
    for _ in range(args.warmup):
        oracle_tokens_per_s(shape, host, n)
    t0 = time.perf_counter()
    total = 0
    for _ in range(args.steps):
        m, _, threads = oracle_tokens_per_s(shape, host, n)
        total += m
    dt = time.perf_counter() - t0
    value = total / dt
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": workload_config(shape, "cpu"),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "host_cores": cores, "cpu_model": model,
                             "sample": f"{n} seeded tokens of the T={shape.T} batch per step (routing, "
                                       f"routed and shared experts, final sum, float64 numpy on one thread)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


FP8_METRIC = "FP8 1x128 activation quantization bandwidth"


def fp8_workload_config(shape: W.LayerShape) -> dict:
    return {"workload": f"{shape.name}: permuted activations [T*K={shape.T * shape.K}, d={shape.d}] bf16, "
                        f"1x128 groups", "l2": "input larger than L2 (no flush)"}


def run_reference_fp8(args):
    """The FP8 oracle (float64 numpy) quantizing a bounded sample of the rows each step."""
    import oracle.fp8 as F8
    shape = W.CONFIGS[args.config]
    cols = shape.d
    groups = -(-cols // 128)
    n = max(1, min(shape.T * shape.K, args.cpu_sample))
    x = W.normal_bf16(shape.seed, 40, 0, (n, cols), 1.0).float().numpy().astype(np.float64)
    for _ in range(args.warmup):
        F8.quantize_rows(x)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        F8.quantize_rows(x)
    dt = time.perf_counter() - t0
    value = args.steps * n * (3 * cols + groups) / dt / 1e9
    line = {"metric": FP8_METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": fp8_workload_config(shape),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"{n} rows of the [{shape.T * shape.K}, {cols}] activations per step "
                                       f"(float64 numpy, per-group loop)"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------

class Ranks:
    """One process per GPU, launched by torchrun: rank and world size from its
    environment, and a process group for the barrier and the max-over-ranks
    time only (the layer has no exchange step; every rank runs a full replica).
    NCCL on GPUs; the tests run the same code over gloo on CPU."""

    def __init__(self, backend: str = "nccl", device=None, timeout_s: float = 120.0):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = device if device is not None else torch.device("cpu")
        self.dist = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
            if backend == "nccl":
                kw["device_id"] = self.device
            dist.init_process_group(backend, **kw)
            self.dist = dist

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max(self, v: float) -> float:
        """The largest of the ranks' values (every rank gets it)."""
        if self.dist is None:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist is not None:
            self.dist.barrier()
            self.dist.destroy_process_group()
            self.dist = None


def aggregate_rate(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return world * units_per_rank / (max_ms * 1e-3)


def device_layer_inputs(shape: W.LayerShape, dev):
    """(host inputs, device inputs) of a layer.  Routed experts are generated one at a time on the
    host's cores and copied straight into stacked device tensors, so a large layer (V3: 22.5 GB of
    expert weights) is never held whole in host memory."""
    from concurrent.futures import ThreadPoolExecutor
    host = W.layer_inputs(shape, with_experts=False)
    d_in = to_device(host, dev)
    N, I, d = shape.N, shape.I, shape.d
    wg = torch.empty((N, I, d), dtype=torch.bfloat16, device=dev)
    wu = torch.empty((N, I, d), dtype=torch.bfloat16, device=dev)
    wd = torch.empty((N, d, I), dtype=torch.bfloat16, device=dev)
    with ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
        for e, (g, u, dn) in enumerate(ex.map(lambda e: W.expert_weights(shape, e), range(N))):
            wg[e].copy_(g)
            wu[e].copy_(u)
            wd[e].copy_(dn)
    d_in["w_gate"], d_in["w_up"], d_in["w_down"] = wg, wu, wd
    return host, d_in


def choose_peak(peaks: dict, timed_s: float, clk) -> tuple:
    """(bf16 TFLOP/s, its name): the burst figure for a short timed region that held the maximum SM
    clock, the sustained (power-capped) one for a long region or a clock below its maximum."""
    at_max = clk is not None and clk.get("sm_mhz", 0) >= 0.97 * clk.get("sm_max_mhz", 1) \
        and "sw_power_cap" not in clk.get("reasons", [])
    if timed_s < 1.0 and (clk is None or at_max):
        return float(peaks["bf16_tflops"]), "bf16_tflops"
    return float(peaks["bf16_tflops_sustained"]), "bf16_tflops_sustained"


def touched_weight_bytes(shape: W.LayerShape, counts, fp8: bool = False) -> dict:
    """Expert weights each GEMM launch must stream: every routed expert that received a token, and
    the shared experts (gate/up: W_gate and W_up; down: W_down); bf16, or FP8 codes with one scale
    byte per 128 x 128 block."""
    touched = int(sum(1 for c in counts if c > 0))
    per_elem = (1.0 + 1.0 / (128 * 128)) if fp8 else 2.0
    per_proj = per_elem * shape.d * (touched * shape.I + shape.Ks * shape.Is)
    return {"touched_experts": touched, "gate_up": 2 * per_proj, "down": per_proj, "layer": 3 * per_proj}


def measure_layer(B, shape: W.LayerShape, host: dict, d_in: dict, dev, local: int, ranks, steps: int,
                  warmup: int, with_e2e: bool, fp8: bool = False):
    """Time `steps` forwards of one layer on its resident inputs (CUDA events on the launching stream,
    barrier + synchronize on both sides, max over ranks), then the same `steps` forwards again with
    events around the dominant kernel (its duration for the roofline), then every kernel in a separate
    pass, then (optionally) the host-buffer entry point.  The step time comes from the region without
    kernel events: an event between two launches ends the early start of the second (programmatic
    dependent launch), which the small batches rely on (16B decode: 0.104 vs 0.114 ms per step).
    fp8: the FP8 layer (moe_forward_fp8) on weights block-quantized by the library beforehand (not
    timed)."""
    world = ranks.world
    layer = B.MoELayer(d_model=shape.d, n_routed=shape.N, d_ff=shape.I, n_shared=shape.Ks,
                       d_ff_shared=shape.Is, max_tokens=shape.T, max_k=shape.K, gate=shape.gate,
                       device=local, flags=B.MOE_FLAG_FP8 if fp8 else 0)
    shared = (d_in["ws_gate"], d_in["ws_up"], d_in["ws_down"]) if shape.Ks else None
    layer.set_weights(d_in["router"], (d_in["w_gate"], d_in["w_up"], d_in["w_down"]), shared,
                      logit_bias=d_in["logit_bias"], select_bias=d_in["select_bias"])
    if fp8:
        layer.set_weights_fp8(tuple(B.quantize_fp8_blocks(d_in[k]) for k in ("w_gate", "w_up", "w_down")),
                              tuple(B.quantize_fp8_blocks(d_in[k]) for k in ("ws_gate", "ws_up", "ws_down"))
                              if shape.Ks else None)
    fwd = layer.forward_fp8 if fp8 else layer.forward
    x = d_in["x"]
    out = torch.empty_like(x)
    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        fwd(x, shape.K, out)
    st = layer.status()
    if st != B.MOE_OK:
        raise B.MoEError(st, f"{shape.name} warm-up")

    clocks = ClockSampler(local)
    time.sleep(0.3)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ranks.barrier()
    torch.cuda.synchronize(dev)
    start.record(stream)
    for _ in range(steps):
        fwd(x, shape.K, out)
    end.record(stream)
    torch.cuda.synchronize(dev)
    ranks.barrier()
    clk = clocks.stop()
    st = layer.status()
    if st != B.MOE_OK:
        raise B.MoEError(st, f"{shape.name} timed region")
    ms_total = ranks.max(start.elapsed_time(end))
    # the same forwards with CUDA events around the dominant kernel only (its own stream), for the roofline
    layer.set_timing(True, kernels=[DOMINANT])
    ranks.barrier()
    torch.cuda.synchronize(dev)
    for _ in range(steps):
        fwd(x, shape.K, out)
    torch.cuda.synchronize(dev)
    ranks.barrier()
    ktimes = layer.kernel_times()
    layer.set_timing(False)
    st = layer.status()
    if st != B.MOE_OK:
        raise B.MoEError(st, f"{shape.name} dominant-kernel region")
    # every kernel's time, and the launches of one forward, from a short pass outside the timed region
    pass_steps = max(1, min(steps, 50))
    layer.set_timing(True)
    for _ in range(pass_steps):
        fwd(x, shape.K, out)
    all_ktimes = layer.kernel_times()
    layer.set_timing(False)
    r = {"ms_total": ms_total, "ms_step": ms_total / steps, "clocks": clk,
         "dominant_ms": ranks.max(ktimes[DOMINANT][0] / max(1, ktimes[DOMINANT][1])),
         "kernel_ms": {k: (v[0] / v[1] if v[1] else 0.0) for k, v in all_ktimes.items()},
         "launches_per_forward": sum(n for _, n in all_ktimes.values()) / pass_steps,
         # per-expert loads of the timed forwards (before any chunked host-buffer forward overwrites them)
         "counts": layer.routing(shape.T, shape.K)[2].cpu().tolist()}
    r["value"] = aggregate_rate(shape.T, world, r["ms_step"])

    if with_e2e:
        x_h = host["x"].pin_memory()
        out_h = torch.empty_like(x_h).pin_memory()
        e2e_steps = max(1, min(steps, 100))
        if fp8:
            # pinned x in, moe_forward_fp8, the output back: all on the stream, the read synchronised
            xd = torch.empty_like(x)

            def host_step():
                xd.copy_(x_h, non_blocking=True)
                layer.forward_fp8(xd, shape.K, out)
                out_h.copy_(out, non_blocking=True)
                torch.cuda.current_stream(dev).synchronize()
        else:
            def host_step():
                layer.forward_host(x_h, shape.K, out_h)
        for _ in range(3):
            host_step()
        ranks.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            host_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ranks.barrier()
        e2e_ms = ranks.max(e0.elapsed_time(e1)) / e2e_steps
        r["e2e"] = {"value": aggregate_rate(shape.T, world, e2e_ms), "unit": UNIT,
                    "h2d_bytes_per_step": int(x_h.numel() * 2), "d2h_bytes_per_step": int(out_h.numel() * 2),
                    "ms_per_step": e2e_ms}
    layer.close()
    return r


def measure_training_step(B, shape: W.LayerShape, d_in: dict, dev, local: int, ranks, warmup: int,
                          fwd_ms: float, peaks: dict, peak_src: str, steps: int = 0) -> dict:
    """The layer's training step on the headline workload: moe_forward, then moe_backward for a seeded
    upstream gradient dh, with every gradient asked for (dx, the gates', the router's and the expert
    and shared weights' in fp32).  Timed like the forward (CUDA events on the launching stream over
    at least ~0.5 s unless `steps` fixes the count, barrier + synchronize on both sides, max over ranks).  Algorithmic FLOPs: the
    forward's, plus twice them for the backward (each GEMM of the forward has one for its input and
    one for its weights); the backward also recomputes the gate/up GEMM (executed FLOPs, reported
    beside them)."""
    world = ranks.world
    layer = B.MoELayer(d_model=shape.d, n_routed=shape.N, d_ff=shape.I, n_shared=shape.Ks,
                       d_ff_shared=shape.Is, max_tokens=shape.T, max_k=shape.K, gate=shape.gate, device=local)
    shared = (d_in["ws_gate"], d_in["ws_up"], d_in["ws_down"]) if shape.Ks else None
    layer.set_weights(d_in["router"], (d_in["w_gate"], d_in["w_up"], d_in["w_down"]), shared,
                      logit_bias=d_in["logit_bias"], select_bias=d_in["select_bias"])
    x = d_in["x"]
    out, dx = torch.empty_like(x), torch.empty_like(x)
    dh = W.output_gradient(shape).to(dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        layer.forward(x, shape.K, out)
        layer.backward(x, shape.K, dh, dx=dx, router_grad=True, weight_grads=True)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    est = time.perf_counter()
    step()
    torch.cuda.synchronize(dev)
    if steps <= 0:
        steps = max(10, int(0.5 / max(time.perf_counter() - est, 1e-6)))
    st = layer.status()
    if st != B.MOE_OK:
        raise B.MoEError(st, "training step warm-up")
    clocks = ClockSampler(local)
    time.sleep(0.3)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ranks.barrier()
    torch.cuda.synchronize(dev)
    start.record(stream)
    for _ in range(steps):
        step()
    end.record(stream)
    torch.cuda.synchronize(dev)
    ranks.barrier()
    clk = clocks.stop()
    st = layer.status()
    if st != B.MOE_OK:
        raise B.MoEError(st, "training step timed region")
    ms = ranks.max(start.elapsed_time(end)) / steps
    layer.close()
    fwd_flop = layer_flop(shape)
    alg_flop = 3 * fwd_flop
    executed = alg_flop + 4 * shape.T * shape.d * (shape.K * shape.I + shape.Ks * shape.Is) + shape.router_flop
    peak, peak_name = choose_peak(peaks, ms * steps * 1e-3, clk)
    tflops = world * alg_flop / (ms * 1e-3) / 1e12
    return {"workload": workload_config(shape, f"replicas{world}" if world > 1 else "single")["workload"],
            "what": "moe_forward + moe_backward (dx, dgate, d_router, d_logit_bias when present, expert and "
                    "shared weight gradients in fp32)",
            "steps": steps, "ms_per_step": ms, "ms_backward": ms - fwd_ms,
            "tokens_per_s": aggregate_rate(shape.T, world, ms),
            "tflops": tflops, "tflops_frac_of_peak": tflops / (world * peak), "tflops_peak": f"{peak_src} {peak_name}",
            "algorithmic_tflop_per_step": alg_flop / 1e12, "executed_tflop_per_step": executed / 1e12,
            "clocks": clk}


def fused_decode(shape: W.LayerShape, fp8: bool = False) -> bool:
    """Whether the layer (bf16 or FP8) runs both expert GEMMs in one launch (the decode FFN)."""
    return shape.T <= DECODE_MAX_T


def roofline_of(shape: W.LayerShape, r: dict, peaks: dict, peak_src: str, traffic=None, fp8: bool = False):
    """Roofline of the dominant kernel (the shared + routed gate/up GEMM with SwiGLU; for a decode
    batch the one launch of both expert GEMMs): tensor-bound when the routed experts' FLOPs per
    weight byte exceed the ridge (sustained bf16 FLOP/s over copy bandwidth), else HBM-bound over the
    weights of the touched experts (the weight-streaming regime).  fp8: the FP8 layer, against twice
    the measured bf16 peak (the nominal FP8 / bf16 ratio of the tensor cores) and over 1-byte weights
    (plus one scale byte per 128 x 128 block)."""
    peak_flops, peak_name = choose_peak(peaks, r["ms_total"] * 1e-3, r["clocks"])
    if fp8:
        peak_flops, peak_name = 2.0 * peak_flops, f"2 x {peak_name} (fp8 = 2 x bf16, nominal ratio)"
    fused = fused_decode(shape, fp8)
    k_flop = (6.0 if fused else 4.0) * shape.T * shape.d * (shape.K * shape.I + shape.Ks * shape.Is)
    wb = touched_weight_bytes(shape, r["counts"], fp8)
    k_bytes = wb["layer"] if fused else wb["gate_up"]
    k_avg_ms = r["dominant_ms"]
    hbm = float(peaks["hbm_gbs"])
    if k_flop / k_bytes > float(peaks["bf16_tflops_sustained"]) * 1e12 / (hbm * 1e9):
        achieved = k_flop / (k_avg_ms * 1e-3) / 1e12
        mult = 2.0 if fp8 else 1.0
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak_flops, "unit": "TFLOP/s",
                "peak_source": f"{peak_src} {peak_name}",
                "frac_of_burst": achieved / (mult * float(peaks["bf16_tflops"])),
                "frac_of_sustained": achieved / (mult * float(peaks["bf16_tflops_sustained"]))}
    else:
        achieved = k_bytes / (k_avg_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "peak_source": f"{peak_src} hbm_gbs"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    if fused:
        kname = (("decode_ffn8_kernel" if fp8 else "decode_ffn_kernel") +
                 " (shared and routed experts: gate/up GEMM + SwiGLU and down GEMM + gate scale, one launch)")
    else:
        kname = ("fp8_gemm_kernel<true>" if fp8 else "gateup_gemm_kernel") + \
            " (shared and routed experts: gate/up GEMM + SwiGLU)"
    roof.update({"traffic": traffic, "kernel": kname, "flop_per_launch": k_flop, "weight_bytes_per_launch": k_bytes,
                 "avg_launch_ms": k_avg_ms})
    return roof, peak_flops, peak_name


def hbm_fractions(shape: W.LayerShape, r: dict, peaks: dict, fp8: bool = False) -> dict:
    """Each expert GEMM's and the whole layer's rate over the touched experts' weight bytes, as a
    fraction of the measured copy bandwidth (the roofline of the weight-streaming shapes)."""
    wb = touched_weight_bytes(shape, r["counts"], fp8)
    hbm = float(peaks["hbm_gbs"])
    out = {"touched_experts": wb["touched_experts"], "weight_bytes": wb["layer"]}
    if fused_decode(shape, fp8):
        ms = r["kernel_ms"].get("gate_up", 0.0)  # both GEMMs in one launch
        out["ffn_gbs"] = wb["layer"] / (ms * 1e-3) / 1e9 if ms > 0 else None
        out["ffn_frac"] = out["ffn_gbs"] / hbm if ms > 0 else None
    else:
        for k in ("gate_up", "down"):
            ms = r["kernel_ms"].get(k, 0.0)
            out[f"{k}_gbs"] = wb[k] / (ms * 1e-3) / 1e9 if ms > 0 else None
            out[f"{k}_frac"] = out[f"{k}_gbs"] / hbm if ms > 0 else None
    out["layer_gbs"] = wb["layer"] / (r["ms_step"] * 1e-3) / 1e9
    out["layer_frac"] = out["layer_gbs"] / hbm
    return out


PER_CONFIG = ("2b", "16b_decode", "v3")


def estimate_step_s(B, shape: W.LayerShape, d_in: dict, dev, local: int) -> float:
    """Seconds per forward of a layer, from 3 warm forwards (outside any timed region)."""
    layer = B.MoELayer(d_model=shape.d, n_routed=shape.N, d_ff=shape.I, n_shared=shape.Ks,
                       d_ff_shared=shape.Is, max_tokens=shape.T, max_k=shape.K, gate=shape.gate, device=local)
    shared = (d_in["ws_gate"], d_in["ws_up"], d_in["ws_down"]) if shape.Ks else None
    layer.set_weights(d_in["router"], (d_in["w_gate"], d_in["w_up"], d_in["w_down"]), shared,
                      logit_bias=d_in["logit_bias"], select_bias=d_in["select_bias"])
    out = torch.empty_like(d_in["x"])
    layer.forward(d_in["x"], shape.K, out)
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    for _ in range(3):
        layer.forward(d_in["x"], shape.K, out)
    torch.cuda.synchronize(dev)
    dt = (time.perf_counter() - t0) / 3
    layer.close()
    return dt


def run_ep_emulated(args):
    """One JSON line: the expert-parallel forward with G ranks emulated on one GPU (G handles whose
    kernels address each other's workspaces, the steps of all ranks in order on one stream, so the
    time is the sum of the ranks' kernels and no NVLink transfer is measured), beside the single-GPU
    layer on the same T tokens.  The V3 workload routes each token to at most 4 ranks when G = 8."""
    from fine_grained_shared_b200 import moe as B

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    shape = W.CONFIGS[args.config]
    G = args.ep_emulate
    if G < 2 or shape.N % G or shape.T % G:
        raise SystemExit(f"--ep-emulate {G}: needs G >= 2 dividing mN = {shape.N} and T = {shape.T}")
    node_limit = (8, 4) if (shape.name == "v3" and G == 8) else None
    host, d_in = device_layer_inputs(shape, dev)
    Tr, per = shape.T // G, shape.N // G
    xs = [d_in["x"][r * Tr:(r + 1) * Tr] for r in range(G)]
    shared = (d_in["ws_gate"], d_in["ws_up"], d_in["ws_down"]) if shape.Ks else None
    layers = []
    for r in range(G):
        layer = B.ExpertParallelLayer(ep_ranks=G, ep_rank=r, d_model=shape.d, n_routed=shape.N, d_ff=shape.I,
                                      n_shared=shape.Ks, d_ff_shared=shape.Is, max_tokens=Tr, max_k=shape.K,
                                      gate=shape.gate, node_limit=node_limit)
        sl = slice(r * per, (r + 1) * per)
        layer.set_weights(d_in["router"], (d_in["w_gate"][sl], d_in["w_up"][sl], d_in["w_down"][sl]), shared,
                          logit_bias=d_in["logit_bias"], select_bias=d_in["select_bias"])
        layers.append(layer)
    B.connect_emulated(layers)
    single = B.MoELayer(d_model=shape.d, n_routed=shape.N, d_ff=shape.I, n_shared=shape.Ks, d_ff_shared=shape.Is,
                        max_tokens=shape.T, max_k=shape.K, gate=shape.gate, node_limit=node_limit)
    single.set_weights(d_in["router"], (d_in["w_gate"], d_in["w_up"], d_in["w_down"]), shared,
                       logit_bias=d_in["logit_bias"], select_bias=d_in["select_bias"])
    outs = [torch.empty_like(x) for x in xs]
    out1 = torch.empty_like(d_in["x"])
    warmup, steps = max(3, args.warmup), max(3, args.steps)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            fn()
        b.record()
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / steps
    clocks = ClockSampler(0)
    time.sleep(0.3)
    ms_ep = timed(lambda: B.forward_emulated(layers, xs, shape.K, outs))
    ms_1 = timed(lambda: single.forward(d_in["x"], shape.K, out1))
    clk = clocks.stop()
    for layer in layers:
        st = layer.status()
        if st != B.MOE_OK:
            raise B.MoEError(st, "expert-parallel forward")
    same = all(torch.equal(outs[r].view(torch.int16), out1[r * Tr:(r + 1) * Tr].view(torch.int16))
               for r in range(G)) if Tr > 256 or shape.T <= 256 else None
    line = {"metric": "MoE layer fwd tokens/s, expert-parallel ranks emulated on one GPU", "value": shape.T / (ms_ep * 1e-3),
            "unit": UNIT, "n_gpus": 1, "ep_ranks_emulated": G, "steps": steps, "warmup": warmup,
            "ms_per_step": ms_ep, "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": workload_config(shape, f"ep{G}-emulated"),
            "single_gpu_ms_per_step": ms_1, "node_limit": node_limit,
            "bit_identical_to_single_gpu": same, "clocks": clk}
    print(json.dumps(line), flush=True)
    for layer in layers:
        layer.close()
    single.close()


def run_training_step(args):
    """One JSON line for the layer's training step alone (moe_forward + moe_backward) on --config."""
    from fine_grained_shared_b200 import moe as B

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    shape = W.CONFIGS[args.config]
    host = host_inputs(shape)
    d_in = to_device(host, dev)
    peaks, peak_src = measured_peaks()
    fwd = measure_layer(B, shape, host, d_in, dev, local, ranks, max(3, args.steps), max(3, args.warmup),
                        with_e2e=False)
    t = measure_training_step(B, shape, d_in, dev, local, ranks, max(3, args.warmup), fwd["ms_step"], peaks, peak_src,
                              steps=args.steps)
    line = {"metric": "MoE layer training step (forward + backward) tokens/s", "value": t["tokens_per_s"],
            "unit": UNIT, "n_gpus": ranks.world, "steps": t["steps"], "warmup": max(3, args.warmup),
            "ms_per_step": t["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": workload_config(shape, f"replicas{ranks.world}" if ranks.world > 1 else "single"),
            "forward_ms_per_step": fwd["ms_step"], "training_step": t}
    if ranks.rank == 0:
        print(json.dumps(line), flush=True)
    ranks.close()


def run_ours(args):
    from fine_grained_shared_b200 import moe as B

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    world, rank = ranks.world, ranks.rank
    warmup = max(3, args.warmup)

    shape = W.CONFIGS[args.config]
    fp8 = args.fp8
    host = host_inputs(shape)
    d_in = to_device(host, dev)
    r = measure_layer(B, shape, host, d_in, dev, local, ranks, args.steps, warmup, with_e2e=True, fp8=fp8)
    del d_in
    torch.cuda.empty_cache()

    peaks, peak_src = measured_peaks()
    roofline, peak_flops, peak_name = roofline_of(shape, r, peaks, peak_src, profiled_traffic(shape, fp8=fp8), fp8)
    layer_tflops = world * layer_flop(shape) / (r["ms_step"] * 1e-3) / 1e12
    config = workload_config(shape, f"replicas{world}" if world > 1 else "single")
    if fp8:
        config["expert_gemms"] = ("fp8: E4M3 operands, 1x128 activation and 128x128 weight scales (UE8M0), "
                                  "fp32 accumulation; router in bf16/fp32")
    line = {
        "metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": warmup, "ms_per_step": r["ms_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp8-e4m3" if fp8 else "bf16", "data": "synthetic",
        "config": config,
        "tflops": layer_tflops,
        "tflops_frac_of_peak": layer_tflops / (world * peak_flops),
        "tflops_peak": f"{peak_src} {peak_name}",
        "roofline": roofline,
        "kernel_ms_per_step": r["kernel_ms"],
        "e2e": r["e2e"],
        "gpu_launches": int(round(r["launches_per_forward"] * args.steps)),
        "clocks": r["clocks"],
    }
    if roofline["bound"] == "hbm":
        line["hbm"] = hbm_fractions(shape, r, peaks, fp8)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(shape, host, fp8=fp8)

    # the layer's training step (forward + backward) on the same workload, after the headline
    if not args.no_per_config and not fp8 and not fused_decode(shape):
        d_in = to_device(host, dev)
        line["training_step"] = measure_training_step(B, shape, d_in, dev, local, ranks, warmup, r["ms_step"],
                                                      peaks, peak_src)
        del d_in
        torch.cuda.empty_cache()

    # the other single-GPU workloads, measured after the headline one: ms per step, tokens/s and the
    # roofline that bounds each (tensor for the 2B layer, HBM over the touched experts' weights for
    # the 16B decode and V3 layers)
    if not args.no_per_config and not fp8:
        per = {}
        for name in PER_CONFIG:
            if name == args.config:
                continue
            cs = W.CONFIGS[name]
            t0 = time.perf_counter()
            chost, cdev = device_layer_inputs(cs, dev)
            gen_s = time.perf_counter() - t0
            # each workload is timed over at least ~0.5 s of forwards, so that the clock sampler
            # (one sample per 100 ms) sees the timed region; the warm-up gives the step time
            steps = max(args.steps, int(0.5 / max(estimate_step_s(B, cs, cdev, dev, local), 1e-6)))
            cr = measure_layer(B, cs, chost, cdev, dev, local, ranks, steps, warmup, with_e2e=False)
            del cdev
            torch.cuda.empty_cache()
            croof, cpeak, cpeak_name = roofline_of(cs, cr, peaks, peak_src, profiled_traffic(cs))
            ctf = world * layer_flop(cs) / (cr["ms_step"] * 1e-3) / 1e12
            per[name] = {"workload": workload_config(cs, f"replicas{world}" if world > 1 else "single")["workload"],
                         "steps": steps, "ms_per_step": cr["ms_step"], "tokens_per_s": cr["value"],
                         "tflops": ctf, "tflops_frac_of_peak": ctf / (world * cpeak),
                         "tflops_peak": f"{peak_src} {cpeak_name}", "roofline": croof,
                         "hbm": hbm_fractions(cs, cr, peaks), "kernel_ms_per_step": cr["kernel_ms"],
                         "clocks": cr["clocks"], "l2": l2_note(cs), "input_generation_s": gen_s}
            line["gpu_launches_per_config"] = line.get("gpu_launches_per_config", 0) + \
                int(round(cr["launches_per_forward"] * steps))
        line["per_config"] = per
    if rank == 0:
        print(json.dumps(line), flush=True)
    ranks.close()


def run_fp8_quant(args):
    """One step = the FP8 1 x 128 quantization of the permuted activations of one forward of the
    workload ([T * K, d] bf16, larger than L2: 403 MB for the 16B prefill layer) through the C ABI.
    The 128 x 128 block quantization of the routed experts' W_gate is timed beside it.  Both kernels
    stream (2 B read, 1 B + 1/128 B written per element): the roofline is HBM bandwidth."""
    from ctypes import c_void_p
    from fine_grained_shared_b200 import moe as B

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    world, rank = ranks.world, ranks.rank
    shape = W.CONFIGS[args.config]
    rows, cols = shape.T * shape.K, shape.d
    groups = -(-cols // 128)
    x_h = W.normal_bf16(shape.seed, 40, 0, (rows, cols), 1.0)
    x = x_h.to(dev)
    q = torch.empty((rows, cols), dtype=torch.uint8, device=dev)
    sc = torch.empty((rows, groups), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = c_void_p(stream.cuda_stream)

    def step(src):
        st = B.moe_quantize_fp8_rows(c_void_p(src.data_ptr()), rows, cols, c_void_p(q.data_ptr()),
                                     c_void_p(sc.data_ptr()), sp)
        if st != B.MOE_OK:
            raise B.MoEError(st, "moe_quantize_fp8_rows")

    for _ in range(max(3, args.warmup)):
        step(x)
    clocks = ClockSampler(local)
    time.sleep(0.3)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ranks.barrier()
    torch.cuda.synchronize(dev)
    start.record(stream)
    for _ in range(args.steps):
        step(x)
    end.record(stream)
    torch.cuda.synchronize(dev)
    ranks.barrier()
    clk = clocks.stop()
    ms_step = ranks.max(start.elapsed_time(end)) / args.steps
    step_bytes = rows * cols * 3 + rows * groups
    value = world * step_bytes / (ms_step * 1e-3) / 1e9

    # end to end: pinned host activations in, codes and scales back to pinned host memory
    xp = x_h.pin_memory()
    qh = torch.empty((rows, cols), dtype=torch.uint8).pin_memory()
    sh = torch.empty((rows, groups), dtype=torch.uint8).pin_memory()
    xd = torch.empty_like(x)
    e2e_steps = max(1, min(args.steps, 20))
    ranks.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        xd.copy_(xp, non_blocking=True)
        step(xd)
        qh.copy_(q, non_blocking=True)
        sh.copy_(sc, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ranks.barrier()
    e2e_ms = ranks.max(e0.elapsed_time(e1)) / e2e_steps

    # the routed experts' W_gate in 128 x 128 blocks, beside it
    w = W.normal_bf16(shape.seed, 3, 0, (shape.N, shape.I, shape.d), shape.sigma).to(dev)
    wq = torch.empty(w.shape, dtype=torch.uint8, device=dev)
    ws = torch.empty((shape.N, -(-shape.I // 128), groups), dtype=torch.uint8, device=dev)

    def wstep():
        st = B.moe_quantize_fp8_blocks(c_void_p(w.data_ptr()), shape.N, shape.I, shape.d,
                                       c_void_p(wq.data_ptr()), c_void_p(ws.data_ptr()), sp)
        if st != B.MOE_OK:
            raise B.MoEError(st, "moe_quantize_fp8_blocks")

    for _ in range(3):
        wstep()
    torch.cuda.synchronize(dev)
    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0.record(stream)
    for _ in range(10):
        wstep()
    w1.record(stream)
    torch.cuda.synchronize(dev)
    w_ms = w0.elapsed_time(w1) / 10
    w_bytes = w.numel() * 3 + ws.numel()

    peaks, peak_src = measured_peaks()
    achieved = step_bytes / (ms_step * 1e-3) / 1e9
    line = {
        "metric": FP8_METRIC, "value": value, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16->e4m3",
        "data": "synthetic",
        "config": fp8_workload_config(shape),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                     "frac": achieved / float(peaks["hbm_gbs"]),
                     "traffic": profiled_traffic(shape, FP8_PROFILES.get(shape.name, ""), FP8_SOURCES)
                     if shape.name in FP8_PROFILES else None,
                     "peak_source": f"{peak_src} hbm_gbs", "kernel": "quantize_rows_kernel",
                     "bytes_per_launch": step_bytes},
        "weights_128x128": {"matrices": f"W_gate [{shape.N}, {shape.I}, {shape.d}]", "ms": w_ms,
                            "gbs": w_bytes / (w_ms * 1e-3) / 1e9,
                            "frac": w_bytes / (w_ms * 1e-3) / 1e9 / float(peaks["hbm_gbs"])},
        "e2e": {"value": world * step_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": rows * cols * 2, "d2h_bytes_per_step": rows * cols + rows * groups,
                "ms_per_step": e2e_ms},
        "gpu_launches": args.steps,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle.fp8 as F8
        n = 512
        xs = x_h[:n].float().numpy().astype(np.float64)
        t0 = time.perf_counter()
        F8.quantize_rows(xs)
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": n * (cols * 3 + groups) / dt / 1e9, "unit": "GB/s", "cores": 1,
                                "kind": "oracle", "sample": f"{n} rows of the [{rows}, {cols}] activations "
                                                            "(float64 numpy, per-group loop)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    ranks.close()


def main():
    args = parse_args()
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return
        run_reference_fp8(args) if args.fp8_quant else run_reference(args)
    elif args.fp8_quant:
        run_fp8_quant(args)
    elif args.training_step:
        run_training_step(args)
    elif args.ep_emulate:
        run_ep_emulated(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
