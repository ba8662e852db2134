#!/usr/bin/env python
"""Benchmark of the MXFP8 W8A8 linear layer on B200.

One step = one pass of the whole hot path over one batch: dynamic MX
quantization of the BF16 activations (one kernel) and the block-scaled
tcgen05 GEMM with the F16-bias / BF16 epilogue (one kernel).  Weights are
quantized once, offline, before timing.  Default workload: the Wan2.2 A14B
self-attention Q projection at 480x832, 81 frames (M = 32760 tokens,
K = N = 5120).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

Prints ONE JSON line (rank 0).  `value` is whole-job TFLOP/s (2*M*N*K per
step per GPU, all GPUs, divided by the slowest rank's device time).  Under
torchrun each rank runs an independent replica (weak scaling, no data-path
collective).  `--impl reference` times the CPU oracle on host cores on a
bounded sample of the same workload.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "MXFP8 W8A8 linear TFLOPS at Wan shapes, % of dense FP8 peak; quant GB/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FP8_OVER_BF16 = 2.0  # nominal dense ratio: 4.5 PF/s FP8 vs 2.25 PF/s BF16
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="c1_q_proj_480p",
                    choices=["c0_small", "c1_q_proj_480p", "ffn0_832x1104", "ffn2_832x1104"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    return ap.parse_args()


def workload_shape(name):
    from mxfp8_w8a8_quantized_b200 import synth
    if name == "c0_small":
        return dict(M=256, K=512, N=512, seed=0, desc="single linear 256x512x512")
    if name == "c1_q_proj_480p":
        return dict(M=synth.TOKENS_480P, K=synth.HIDDEN, N=synth.HIDDEN, seed=1,
                    desc="Wan2.2 A14B attn1.to_q at 480x832, 81 frames (21x30x52 tokens)")
    if name == "ffn0_832x1104":
        return dict(M=synth.TOKENS_832x1104, K=synth.HIDDEN, N=synth.FFN, seed=2,
                    desc="Wan2.2 A14B ffn.net.0.proj at 832x1104, 81 frames")
    if name == "ffn2_832x1104":
        return dict(M=synth.TOKENS_832x1104, K=synth.FFN, N=synth.HIDDEN, seed=2,
                    desc="Wan2.2 A14B ffn.net.2 at 832x1104, 81 frames")
    raise ValueError(name)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


# ---------------------------------------------------------------- distributed
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, v):
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index):
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._h is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples)}


# ---------------------------------------------------------------- our arm
def run_ours(args, world, rank, local):
    from mxfp8_w8a8_quantized_b200 import mxfp8, synth

    shp = workload_shape(args.workload)
    M, K, N, seed = shp["M"], shp["K"], shp["N"], shp["seed"]
    dev = torch.device("cuda", local)
    # synthetic inputs drawn on the device (same recipe as the tests)
    x = synth.activations_device(M, K, seed, 0, dev)
    w = synth.weights_device(N, K, seed, 0, dev)
    b = synth.bias_device(N, seed, 0, dev)
    wq, ws = mxfp8.quantize_weight(w)          # offline weight quantization
    del w
    xq = torch.empty((M, K), dtype=torch.uint8, device=dev)
    xs = torch.empty(mxfp8.scale_bytes(M, K), dtype=torch.uint8, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        mxfp8.quantize(x, codes=xq, scales=xs)
        mxfp8.gemm_prequant(xq, xs, wq, ws, b, out=y)

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if mxfp8.device_status() != 0:
        raise RuntimeError("kernel reported a pipeline timeout during warm-up")

    K_steps = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K_steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(K_steps):
            flush.zero_()                      # L2 flushed between timed steps
            e0, e1, e2 = ev[i]
            e0.record(stream)
            mxfp8.quantize(x, codes=xq, scales=xs)
            e1.record(stream)
            mxfp8.gemm_prequant(xq, xs, wq, ws, b, out=y)
            e2.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    if mxfp8.device_status() != 0:
        raise RuntimeError("kernel reported a pipeline timeout")
    q_ms = [e[0].elapsed_time(e[1]) for e in ev]
    g_ms = [e[1].elapsed_time(e[2]) for e in ev]
    s_ms = [e[0].elapsed_time(e[2]) for e in ev]
    total_ms = max_over_ranks(world, sum(s_ms))
    ms_per_step = total_ms / K_steps
    flops = 2.0 * M * N * K
    value = world * flops * K_steps / (total_ms * 1e-3) / 1e12

    hbm, bf16, peak_src = load_peaks()
    fp8_peak = bf16 * FP8_OVER_BF16
    gemm_ms = statistics.mean(g_ms)
    quant_ms = statistics.mean(q_ms)
    gemm_tflops = flops / (gemm_ms * 1e-3) / 1e12
    quant_bytes = M * K * 2 + M * K + M * K // 32
    quant_gbs = quant_bytes / (quant_ms * 1e-3) / 1e9
    traffic = load_traffic(args.workload)

    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K_steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3 (MXFP8 operands, fp32 accumulate, bf16 out)",
        "data": "synthetic (seeded N(0,1) activations with 1% x20 outlier channels, N(0,1/sqrt(K)) weights, "
                "N(0,0.01) f16 bias)",
        "config": {"workload": args.workload, "desc": shp["desc"], "M": M, "K": K, "N": N,
                   "l2": "flushed between timed steps (256 MiB write outside the step events)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": {"bound": "tensor", "kernel": "mxfp8_gemm_kernel",
                     "achieved": round(gemm_tflops, 1), "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                     "frac": round(gemm_tflops / fp8_peak, 4),
                     "peak_source": f"{peak_src} bf16 burst x {FP8_OVER_BF16} (nominal FP8/BF16 ratio)",
                     "traffic": traffic,
                     "algorithmic_bytes": M * K * (1 + 1 / 32) + N * K * (1 + 1 / 32) + 2 * M * N + 2 * N,
                     "avg_launch_ms": round(gemm_ms, 4)},
        "quant": {"kernel": "mx_quantize_kernel", "achieved_gbs": round(quant_gbs, 1), "peak_gbs": hbm,
                  "frac": round(quant_gbs / hbm, 4), "peak_source": f"{peak_src} copy",
                  "bytes_per_launch": quant_bytes, "avg_launch_ms": round(quant_ms, 4)},
        "gpu_launches": 2 * K_steps,
        "clocks": clk.summary(),
    }
    if not args.no_e2e:
        out["e2e"] = run_e2e(args, mxfp8, x, wq, ws, b, M, K, N, world, dev)
    return out


def run_e2e(args, mxfp8, x_dev, wq, ws, b, M, K, N, world, dev):
    """Same metric through the public API with host buffers: pinned host X ->
    device, mxfp8.linear, Y -> pinned host, all inside the timed region."""
    x_host = torch.empty((M, K), dtype=torch.bfloat16, pin_memory=True)
    x_host.copy_(x_dev.cpu())
    y_host = torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True)
    x_stage = torch.empty_like(x_dev)
    y_dev = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws_buf = torch.empty(mxfp8.linear_workspace_bytes(M, K), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    steps = max(3, min(args.steps, 20))

    def step():
        x_stage.copy_(x_host, non_blocking=True)
        mxfp8.linear(x_stage, wq, ws, b, out=y_dev, workspace=ws_buf)
        y_host.copy_(y_dev, non_blocking=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(world, e0.elapsed_time(e1))
    barrier(world)
    value = world * 2.0 * M * N * K * steps / (ms * 1e-3) / 1e12
    return {"value": round(value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": M * K * 2,
            "d2h_bytes_per_step": M * N * 2, "steps": steps, "ms_per_step": round(ms / steps, 3)}


def load_traffic(workload):
    """dram bytes per GEMM launch from the committed ncu summary, if it is for
    the current kernel build (profiles/<kernel>_<workload>.json)."""
    path = os.path.join(ROOT, "profiles", f"mxfp8_gemm_{workload}.json")
    try:
        d = json.load(open(path))
        from mxfp8_w8a8_quantized_b200 import build
        if d.get("kernel_source_sha") != build.source_sha():
            return None
        return d["dram_bytes_per_launch"]
    except Exception:
        return None


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(shp, rows, seed_rows=0):
    """Inputs of a bounded sample: `rows` rows of X and all of W (quantized
    by the oracle outside the timed region, as the weights are offline)."""
    import numpy as np

    import oracle
    from mxfp8_w8a8_quantized_b200 import synth
    M, K, N, seed = shp["M"], shp["K"], shp["N"], shp["seed"]
    x = synth.activations(rows, K, seed, index=100 + seed_rows)
    w = synth.weights(N, K, seed, index=100)
    b = synth.bias(N, seed, index=100)
    wq, ws = oracle.quantize_f32(w.numpy())
    xb = x.view(torch.int16).numpy().view(np.uint16)
    bb = b.view(torch.int16).numpy().view(np.uint16)
    return xb, wq, ws, bb


def oracle_step(xb, wq, ws, bb):
    import oracle
    xq, xs = oracle.quantize_bf16(xb)
    return oracle.linear(xq, xs, wq, ws, bb)


def cpu_baseline(shp, target_s):
    import oracle
    K, N = shp["K"], shp["N"]
    xb, wq, ws, bb = oracle_sample(shp, 2)
    t0 = time.perf_counter()
    oracle_step(xb, wq, ws, bb)
    t_probe = (time.perf_counter() - t0) / 2
    rows = int(max(1, min(shp["M"], target_s / max(t_probe, 1e-6))))
    xb, wq, ws, bb = oracle_sample(shp, rows)
    t0 = time.perf_counter()
    oracle_step(xb, wq, ws, bb)
    dt = time.perf_counter() - t0
    return {"value": round(2.0 * rows * N * K / dt / 1e12, 6), "unit": "TFLOP/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{rows} of {shp['M']} rows (quantize + FP64 linear over all {N} columns, K={K}); "
                      f"weights quantized outside the timed region; {dt:.1f} s"}


def run_reference(args, world, rank):
    """The oracle as the reference arm: CPU, rank 0 only."""
    import oracle
    shp = workload_shape(args.workload)
    M, K, N = shp["M"], shp["K"], shp["N"]
    if rank != 0:
        return None
    budget = 150.0  # seconds for warm-up + timed steps together
    xb, wq, ws, bb = oracle_sample(shp, 1)
    t0 = time.perf_counter()
    oracle_step(xb, wq, ws, bb)
    t_row = time.perf_counter() - t0
    n_steps = args.steps + args.warmup
    rows = int(max(1, min(M, budget / n_steps / max(t_row, 1e-6))))
    xb, wq, ws, bb = oracle_sample(shp, rows)
    for _ in range(args.warmup):
        oracle_step(xb, wq, ws, bb)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(xb, wq, ws, bb)
    dt = time.perf_counter() - t0
    value = 2.0 * rows * N * K * args.steps / dt / 1e12
    sample = f"{rows} of {M} rows per step (quantize + FP64 linear over all {N} columns, K={K})"
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 6),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (same recipe as the GPU arm)",
        "config": {"workload": args.workload, "desc": shp["desc"], "M": M, "K": K, "N": N},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        out = run_ours(args, world, rank, local)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline(workload_shape(args.workload), args.cpu_seconds)
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
