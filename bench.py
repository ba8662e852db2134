#!/usr/bin/env python
"""Benchmark of the MXFP8 W8A8 linear layer on B200.

One step = one pass of the whole hot path over one batch: dynamic MX
quantization of every BF16 activation and the block-scaled tcgen05 GEMM
with its F16-bias / BF16 epilogue for every linear of the workload (plus the
GELU between the FFN linears).  Weights are quantized once, offline, before
timing.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

Default workload: one denoising step of Wan2.2 A14B at 832x1104, 81 frames
(40 blocks x 10 quantized linears, 75348 video / 512 text tokens), the
largest single-GPU configuration and the one holding both FFN shapes.

Prints ONE JSON line (rank 0).  `value` is whole-job TFLOP/s (2*M*N*K summed
over the step's linears, over all GPUs, divided by the slowest rank's device
time).  Under torchrun every rank runs an independent replica (weak scaling,
no data-path collective).  `--impl reference` times the CPU oracle on host
cores on a bounded sample of the same workload.
"""
import argparse
import json
import os
import statistics
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
FALLBACK_BF16_SUSTAINED = 1400.0
FP8_OVER_BF16 = 2.0  # nominal dense ratio: 4.5 PF/s FP8 vs 2.25 PF/s BF16
FP4_OVER_BF16 = 4.0  # nominal dense ratio: 9 PF/s FP4 vs 2.25 PF/s BF16
L2_FLUSH_BYTES = 256 << 20
WORKLOADS = ["c4_step_832x1104", "c1_q_proj_480p", "c0_small", "ffn0_832x1104", "ffn2_832x1104",
             "c2_ffn_pair_832x1104", "c3_block_832x1104"]


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOADS[0], choices=WORKLOADS)
    ap.add_argument("--unfused", action="store_true",
                    help="chained workloads: separate q/k/v (and text k/v) GEMMs, and ffn.net.0.proj writes "
                         "BF16 with GELU + quantization as separate kernels (default: fused)")
    ap.add_argument("--scheme", choices=["mxfp8", "fp8rowwise", "nvfp4"], default="mxfp8",
                    help="quantization scheme of the single-linear workloads (default: MXFP8)")
    ap.add_argument("--graph", action="store_true",
                    help="capture one step as a CUDA graph and time its replays (per-kernel times then "
                         "come from 3 eager steps)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--reference-seconds", type=float, default=150.0,
                    help="CPU time budget of the reference arm (warm-up + timed steps)")
    return ap.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        burst = float(d["bf16_tflops"])
        return float(d["hbm_gbs"]), burst, float(d.get("bf16_tflops_sustained", burst)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_SUSTAINED, "fallback"


# ---------------------------------------------------------------- ranks
class Ranks:
    """World / rank bookkeeping; collectives only for the barrier and the
    max over ranks (no data-path collective).  Works with NCCL (GPU tensors)
    and gloo (CPU tensors)."""

    def __init__(self, backend=None, device=None):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = device
        self.dist = None
        if self.world > 1 and backend is not None:
            import datetime

            import torch.distributed as dist
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            kw = dict(timeout=datetime.timedelta(seconds=120))
            if backend == "nccl":
                kw["device_id"] = device
            dist.init_process_group(backend, **kw)
            self.dist = dist

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max(self, v: float) -> float:
        if self.dist is None:
            return v
        dev = self.device if (self.device is not None and self.dist.get_backend() == "nccl") else "cpu"
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist is not None:
            self.dist.destroy_process_group()


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


# ---------------------------------------------------------------- timing
def call_label(fn):
    """The linear a call runs, when the callee is a named linear (or one of
    its methods); None otherwise."""
    return getattr(fn, "name", None) or getattr(getattr(fn, "__self__", None), "name", None)


class KernelTimer:
    """CUDA events around each library call of a step, on the launching
    stream: per-kind device time (GEMM, quantizer, GELU), and per linear for
    the GEMMs of named linears."""

    def __init__(self, stream):
        self.stream = stream
        self.events = []          # (kind, label, start, end)
        self.on = False

    def __call__(self, kind, fn, *a, **kw):
        if not self.on:
            return fn(*a, **kw)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(self.stream)
        r = fn(*a, **kw)
        e.record(self.stream)
        self.events.append((kind, call_label(fn), s, e))
        return r

    def totals(self):
        out = {}
        for kind, _, s, e in self.events:
            n, t = out.get(kind, (0, 0.0))
            out[kind] = (n + 1, t + s.elapsed_time(e))
        return out

    def per_label(self, kind="gemm"):
        """{label: (launches, total ms)} over the calls of `kind` that carry a label."""
        out = {}
        for k, label, s, e in self.events:
            if k == kind and label is not None:
                n, t = out.get(label, (0, 0.0))
                out[label] = (n + 1, t + s.elapsed_time(e))
        return out


# ---------------------------------------------------------------- workloads
class LinearWorkload:
    """One quantized linear: Y = BF16(MXFP8(X) MXFP8(W)^T + b)."""

    long_step = False
    scheme = "mxfp8"
    gemm_kernel = "mxfp8_gemm_kernel"
    quant_kernel = "mx_quantize_kernel"
    profile_kernel = "mxfp8_gemm"          # kernel files the profile summary is tied to
    tc_over_bf16 = FP8_OVER_BF16          # tensor-core rate of the GEMM's operand type vs BF16
    dtype = "e4m3 (MXFP8 operands, fp32 accumulate, bf16 out)"

    def __init__(self, name, M, K, N, seed, desc):
        self.name, self.M, self.K, self.N, self.seed, self.desc = name, M, K, N, seed, desc

    @property
    def profile_key(self):
        return self.name if self.scheme == "mxfp8" else f"{self.name}_{self.scheme}"

    def config(self):
        return {"M": self.M, "K": self.K, "N": self.N}

    def linear_flops(self):
        """FLOPs of one launch of each named GEMM (none for a single linear)."""
        return {}

    def flops(self):
        return 2.0 * self.M * self.N * self.K

    def quant_bytes(self):
        return self.M * self.K * (2 + 1) + self.M * self.K // 32

    def gemm_bytes(self):
        M, K, N = self.M, self.K, self.N
        return M * K * (1 + 1 / 32) + N * K * (1 + 1 / 32) + 2 * M * N + 2 * N

    def setup(self, dev):
        from mxfp8_w8a8_quantized_b200 import mxfp8, synth
        self.mx = mxfp8
        M, K, N, s = self.M, self.K, self.N, self.seed
        self.x = synth.activations_device(M, K, s, 0, dev)
        w = synth.weights_device(N, K, s, 0, dev)
        self.b = synth.bias_device(N, s, 0, dev)
        self.wq, self.ws = mxfp8.quantize_weight(w)      # offline weight quantization
        del w
        self.xq = torch.empty((M, K), dtype=torch.uint8, device=dev)
        self.xs = torch.empty(mxfp8.scale_bytes(M, K), dtype=torch.uint8, device=dev)
        self.y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        self.launches = 2

    def step(self, T):
        mx = self.mx
        T("quant", mx.quantize, self.x, codes=self.xq, scales=self.xs)
        T("gemm", mx.gemm_prequant, self.xq, self.xs, self.wq, self.ws, self.b, out=self.y)

    def e2e_io(self):
        return self.x, self.y

    def e2e_step(self, x_dev, y_dev, ws):
        self.mx.linear(x_dev, self.wq, self.ws, self.b, out=y_dev, workspace=ws)

    def e2e_workspace(self, dev):
        return torch.empty(self.mx.linear_workspace_bytes(self.M, self.K), dtype=torch.uint8, device=dev)


def _gemm_bytes(M, K, N, quantized_out=False):
    """Algorithmic HBM bytes of one GEMM launch: operands with their scales,
    bias, and the output (BF16, or E4M3 codes + scales when the epilogue
    quantizes for the next linear)."""
    out = M * N * (1 + 1 / 32) if quantized_out else 2 * M * N
    return M * K * (1 + 1 / 32) + N * K * (1 + 1 / 32) + out + 2 * N


def _quant_bytes(M, K):
    """Algorithmic HBM bytes of one activation quantization."""
    return M * K * 3 + M * K // 32


class FP8RowwiseLinearWorkload(LinearWorkload):
    """One per-channel FP8 linear: FP32 scale per token (dynamic, amax / 448)
    and per output channel; Y = BF16(sx sw (Xq . Wq^T) + b)."""

    scheme = "fp8rowwise"
    quant_kernel = "fp8_rowwise_quantize_bulk_kernel"
    dtype = "e4m3 (per-channel FP8 operands, fp32 accumulate, bf16 out)"

    def config(self):
        return {"M": self.M, "K": self.K, "N": self.N,
                "scheme": "per-channel FP8 (E4M3, FP32 scale per token and per output channel)"}

    def quant_bytes(self):
        return self.M * self.K * 3 + 4 * self.M

    def gemm_bytes(self):
        M, K, N = self.M, self.K, self.N
        return M * K + N * K + 4 * M + 4 * N + 2 * M * N + 2 * N

    def setup(self, dev):
        from mxfp8_w8a8_quantized_b200 import mxfp8, synth
        self.mx = mxfp8
        M, K, N, s = self.M, self.K, self.N, self.seed
        self.x = synth.activations_device(M, K, s, 0, dev)
        w = synth.weights_device(N, K, s, 0, dev)
        self.b = synth.bias_device(N, s, 0, dev)
        self.wq, self.ws = mxfp8.fp8rw_quantize_weight(w)   # offline weight quantization
        del w
        self.xq = torch.empty((M, K), dtype=torch.uint8, device=dev)
        self.xs = torch.empty(M, dtype=torch.float32, device=dev)
        self.y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        self.launches = 2

    def step(self, T):
        mx = self.mx
        T("quant", mx.fp8rw_quantize, self.x, codes=self.xq, scales=self.xs)
        T("gemm", mx.fp8rw_gemm, self.xq, self.xs, self.wq, self.ws, self.b, out=self.y)

    def e2e_step(self, x_dev, y_dev, ws):
        self.mx.fp8rw_linear(x_dev, self.wq, self.ws, self.b, out=y_dev, workspace=ws)

    def e2e_workspace(self, dev):
        return torch.empty(self.mx.fp8rw_linear_workspace_bytes(self.M, self.K), dtype=torch.uint8, device=dev)


class NVFP4LinearWorkload(LinearWorkload):
    """One NVFP4 linear: E2M1 codes with a UE4M3 scale per 16 elements and
    an FP32 global scale per tensor; Y = BF16(alpha (Xh . Wh^T) + b) with
    alpha = 1 / (g_x g_w), formed by the GEMM.  The weights' global scale
    comes from their amax and the activations' from the amax of this
    workload's input, both on the device before timing (the activation
    scale is a calibrated constant of the layer, not computed per step)."""

    scheme = "nvfp4"
    gemm_kernel = "mxfp8_gemm_kernel"     # its NVFP4 mode: tcgen05.mma kind::mxf4nvf4
    quant_kernel = "nvfp4_quantize_kernel"
    profile_kernel = "mxfp8_gemm"
    tc_over_bf16 = FP4_OVER_BF16
    dtype = "e2m1 + ue4m3/16 (NVFP4 operands on the 4-bit block-scaled tensor-core kind), fp32 accumulate, " \
            "bf16 out"

    def config(self):
        return {"M": self.M, "K": self.K, "N": self.N,
                "scheme": "NVFP4 (E2M1, UE4M3 scale per 16, FP32 global scale per tensor)"}

    def quant_bytes(self):
        return self.M * self.K * 2 + self.M * self.K // 2 + self.M * self.K // 16

    def gemm_bytes(self):
        M, K, N = self.M, self.K, self.N
        return (M + N) * K * (1 / 2 + 1 / 16) + 2 * M * N + 2 * N

    def setup(self, dev):
        from mxfp8_w8a8_quantized_b200 import mxfp8, synth
        self.mx = mxfp8
        M, K, N, s = self.M, self.K, self.N, self.seed
        self.x = synth.activations_device(M, K, s, 0, dev)
        w = synth.weights_device(N, K, s, 0, dev)
        self.b = synth.bias_device(N, s, 0, dev)
        self.gw = mxfp8.nvfp4_global_scale(w)           # device tensors; the GEMM forms alpha
        self.gx = mxfp8.nvfp4_global_scale(self.x)
        self.wq, self.ws = mxfp8.nvfp4_quantize_weight(w, self.gw)   # offline weight quantization
        del w
        self.xq = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        self.xs = torch.empty(mxfp8.nvfp4_scale_bytes(M, K), dtype=torch.uint8, device=dev)
        self.y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        self.launches = 2

    def step(self, T):
        mx = self.mx
        T("quant", mx.nvfp4_quantize, self.x, self.gx, codes=self.xq, scales=self.xs)
        T("gemm", mx.nvfp4_gemm, self.xq, self.xs, self.wq, self.ws, self.gx, self.gw, self.b, out=self.y)

    def e2e_step(self, x_dev, y_dev, ws):
        self.mx.nvfp4_linear(x_dev, self.gx, self.wq, self.ws, self.gw, self.b, out=y_dev, workspace=ws)

    def e2e_workspace(self, dev):
        return torch.empty(self.mx.nvfp4_linear_workspace_bytes(self.M, self.K), dtype=torch.uint8, device=dev)


class FFNPairWorkload(LinearWorkload):
    """ffn.net.0.proj -> GELU(tanh) -> ffn.net.2 at M tokens.  Fused (the
    default): ffn.net.0.proj's epilogue applies the GELU and quantizes for
    ffn.net.2; otherwise GEMM, GELU kernel and quantizer run separately."""

    long_step = True

    def __init__(self, name, M, seed, desc, fused=True):
        from mxfp8_w8a8_quantized_b200 import synth
        super().__init__(name, M, synth.HIDDEN, synth.FFN, seed, desc)
        self.fused = fused

    def config(self):
        return {"M": self.M, "hidden": self.K, "ffn": self.N,
                "ffn0_epilogue": "gelu + quantize fused" if self.fused else "bf16 out; gelu, quantize separate"}

    def flops(self):
        return 2 * 2.0 * self.M * self.N * self.K

    def linear_flops(self):
        return {"ffn.net.0.proj": 2.0 * self.M * self.K * self.N, "ffn.net.2": 2.0 * self.M * self.N * self.K}

    def quant_bytes(self):
        q = _quant_bytes(self.M, self.K)
        return q if self.fused else q + _quant_bytes(self.M, self.N)

    def gemm_bytes(self):
        M, H, F = self.M, self.K, self.N
        return _gemm_bytes(M, H, F, quantized_out=self.fused) + _gemm_bytes(M, F, H)

    def setup(self, dev):
        from mxfp8_w8a8_quantized_b200 import mxfp8, synth
        from mxfp8_w8a8_quantized_b200.workloads import QLinear, Workspace
        self.mx = mxfp8
        M, H, F, s = self.M, self.K, self.N, self.seed
        self.x = synth.activations_device(M, H, s, 0, dev)
        self.l0 = QLinear.random(H, F, s, 1, dev)
        self.l2 = QLinear.random(F, H, s, 2, dev)
        self.l0.name, self.l2.name = "ffn.net.0.proj", "ffn.net.2"
        self.wsx = Workspace(M * H, M, H, dev)
        self.wsf = Workspace(M * F, M, F, dev)
        self.f = None if self.fused else torch.empty((M, F), dtype=torch.bfloat16, device=dev)
        self.y = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
        self.launches = 3 if self.fused else 5

    def _run(self, T, x, y):
        mx = self.mx
        xq, xs = T("quant", self.wsx.quantize, x)
        if self.fused:
            fq, fs = T("gemm", self.l0.quantize_out, xq, xs, mx.ACT_GELU_TANH, self.wsf)
        else:
            T("gemm", self.l0, xq, xs, out=self.f)
            T("gelu", mx.gelu_tanh, self.f, out=self.f)
            fq, fs = T("quant", self.wsf.quantize, self.f)
        T("gemm", self.l2, fq, fs, out=y)

    def step(self, T):
        self._run(T, self.x, self.y)

    def e2e_step(self, x_dev, y_dev, ws):
        self._run(lambda k, f, *a, **kw: f(*a, **kw), x_dev, y_dev)

    def e2e_workspace(self, dev):
        return None


class BlocksWorkload(LinearWorkload):
    """`nblocks` Wan blocks (10 quantized linears each) at M video / T text
    tokens; ffn.net.0.proj's epilogue fused with GELU + quantization unless
    fused=False."""

    long_step = True

    def __init__(self, name, M, T, nblocks, seed, desc, fused=True):
        from mxfp8_w8a8_quantized_b200 import synth
        super().__init__(name, M, synth.HIDDEN, synth.FFN, seed, desc)
        self.T, self.nblocks, self.fused = T, nblocks, fused

    def config(self):
        return {"M": self.M, "text_tokens": self.T, "blocks": self.nblocks, "hidden": self.K, "ffn": self.N,
                "projections": "fused qkv (N=15360) and text kv (N=10240)" if self.fused else "separate",
                "ffn0_epilogue": "gelu + quantize fused" if self.fused else "bf16 out; gelu, quantize separate"}

    def _launches(self):
        """The GEMM launches of one block as (rows, K, N, quantized_out) and
        the stand-alone quantizations as (rows, K)."""
        from mxfp8_w8a8_quantized_b200 import synth
        H, F, M, T = self.K, self.N, self.M, self.T
        if self.fused:   # fused QKV / KV projections, GELU + quantize in ffn.net.0.proj
            gemms = [(M, H, 3 * H, False), (M, H, H, False), (M, H, H, False), (T, H, 2 * H, False),
                     (M, H, H, False), (M, H, F, True), (M, F, H, False)]
            quants = [(M, H)] * 5 + [(T, H)]
        else:
            gemms = [(M if kind == "video" else T, K, N, False) for _, K, N, kind in synth.block_linears()]
            quants = [(M, H)] * 5 + [(T, H), (M, F)]
        return gemms, quants

    def linear_flops(self):
        """FLOPs of one launch of each named GEMM of a block."""
        H, F, M, T = self.K, self.N, self.M, self.T
        if self.fused:
            out = {"attn1.to_qkv": 2.0 * M * H * 3 * H, "attn2.to_kv": 2.0 * T * H * 2 * H}
        else:
            out = {n: 2.0 * M * H * H for n in ("attn1.to_q", "attn1.to_k", "attn1.to_v")}
            out.update({n: 2.0 * T * H * H for n in ("attn2.to_k", "attn2.to_v")})
        out.update({"attn1.to_out": 2.0 * M * H * H, "attn2.to_q": 2.0 * M * H * H, "attn2.to_out": 2.0 * M * H * H,
                    "ffn.net.0.proj": 2.0 * M * H * F, "ffn.net.2": 2.0 * M * F * H})
        return out

    def _per_block(self):
        gemms, quants = self._launches()
        fl = sum(2.0 * r * K * N for r, K, N, _ in gemms)
        gb = sum(_gemm_bytes(r, K, N, quantized_out=q) for r, K, N, q in gemms)
        qb = sum(_quant_bytes(r, K) for r, K in quants)
        return fl, qb, gb

    def flops(self):
        return self.nblocks * self._per_block()[0]

    def quant_bytes(self):
        return self.nblocks * self._per_block()[1]

    def gemm_bytes(self):
        return self.nblocks * self._per_block()[2]

    def setup(self, dev):
        from mxfp8_w8a8_quantized_b200 import mxfp8, synth
        from mxfp8_w8a8_quantized_b200.workloads import Block, workspaces
        self.mx = mxfp8
        s = self.seed
        self.x = synth.activations_device(self.M, self.K, s, 1000, dev)
        self.ctx = synth.activations_device(self.T, self.K, s, 1001, dev)
        self.blocks = [Block(s, b, dev) for b in range(self.nblocks)]
        self.wa, self.wb = workspaces(self.M, self.T, dev)
        self.y = None
        gemms, quants = self._launches()
        self.launches = self.nblocks * (len(gemms) + len(quants) + (0 if self.fused else 1))

    def _run(self, T, x):
        y = x
        for blk in self.blocks:
            y = blk.forward(y, self.ctx, self.wa, self.wb, fuse_qkv=self.fused, fuse_ffn=self.fused, timer=T)
        return y

    def step(self, T):
        self.y = self._run(T, self.x)

    def e2e_io(self):
        return self.x, torch.empty_like(self.x)

    def e2e_step(self, x_dev, y_dev, ws):
        y_dev.copy_(self._run(lambda k, f, *a, **kw: f(*a, **kw), x_dev))

    def e2e_workspace(self, dev):
        return None


def make_workload(name, fused=True, scheme="mxfp8"):
    from mxfp8_w8a8_quantized_b200 import synth
    if scheme in ("fp8rowwise", "nvfp4"):
        wl = make_workload(name)
        if type(wl) is not LinearWorkload:
            raise ValueError(f"the {scheme} scheme is measured on the single-linear workloads")
        cls = FP8RowwiseLinearWorkload if scheme == "fp8rowwise" else NVFP4LinearWorkload
        return cls(wl.name, wl.M, wl.K, wl.N, wl.seed, wl.desc)
    H, F = synth.HIDDEN, synth.FFN
    M1, M2, T = synth.TOKENS_480P, synth.TOKENS_832x1104, synth.TEXT_TOKENS
    if name == "c0_small":
        return LinearWorkload(name, 256, 512, 512, 0, "single linear 256x512x512")
    if name == "c1_q_proj_480p":
        return LinearWorkload(name, M1, H, H, 1, "Wan2.2 A14B attn1.to_q at 480x832, 81 frames (21x30x52 tokens)")
    if name == "ffn0_832x1104":
        return LinearWorkload(name, M2, H, F, 2, "Wan2.2 A14B ffn.net.0.proj at 832x1104, 81 frames")
    if name == "ffn2_832x1104":
        return LinearWorkload(name, M2, F, H, 2, "Wan2.2 A14B ffn.net.2 at 832x1104, 81 frames")
    if name == "c2_ffn_pair_832x1104":
        return FFNPairWorkload(name, M2, 2, "Wan2.2 A14B FFN pair (5120->13824->5120, GELU-tanh) at 832x1104",
                               fused=fused)
    if name == "c3_block_832x1104":
        return BlocksWorkload(name, M2, T, 1, 3, "one Wan2.2 A14B block's 10 quantized linears at 832x1104",
                              fused=fused)
    if name == "c4_step_832x1104":
        return BlocksWorkload(name, M2, T, synth.BLOCKS, 4,
                              "one denoising step: 40 blocks x 10 quantized linears at 832x1104", fused=fused)
    raise ValueError(name)


def run_config(wl, world):
    """The `config` object of the JSON line; both arms print the same one."""
    return dict(workload=wl.name, desc=wl.desc, **wl.config(),
                parallelism=f"replicas x{world}" if world > 1 else "single GPU")


# ---------------------------------------------------------------- our arm
def run_ours(args, ranks, dev):
    wl = make_workload(args.workload, fused=not args.unfused, scheme=args.scheme)
    wl.setup(dev)
    stream = torch.cuda.current_stream(dev)
    mx = wl.mx
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    T = KernelTimer(stream)
    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        wl.step(T)
    torch.cuda.synchronize()
    if mx.device_status() != 0:
        raise RuntimeError("kernel reported a pipeline timeout during warm-up")

    steps = args.steps
    graph = None
    if args.graph:
        from mxfp8_w8a8_quantized_b200.workloads import StepGraph
        graph = StepGraph(lambda: wl.step(T))   # T is off: no events inside the graph
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    T.on = graph is None
    ranks.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index or 0) as clk:
        for i in range(steps):
            flush.zero_()                      # L2 flushed between timed steps
            ev[i][0].record(stream)
            if graph is not None:
                graph.replay()
            else:
                wl.step(T)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    ranks.barrier()
    if mx.device_status() != 0:
        raise RuntimeError("kernel reported a pipeline timeout")
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = ranks.max(sum(step_ms))
    ms_per_step = total_ms / steps
    value = ranks.world * wl.flops() * steps / (total_ms * 1e-3) / 1e12
    kernel_steps = steps
    if graph is not None:
        # per-kernel device times come from a few eager steps after the timed
        # graph replays (events cannot sit between a graph's kernels)
        kernel_steps = min(steps, 3)
        T.on = True
        for _ in range(kernel_steps):
            flush.zero_()
            wl.step(T)
        torch.cuda.synchronize()

    hbm, bf16_burst, bf16_sustained, peak_src = load_peaks()
    # a single linear is a kernel timed on its own (burst peak); the chained
    # workloads keep the GPU busy for the whole step (sustained peak)
    kind = "sustained" if wl.long_step else "burst"
    tc_peak = (bf16_sustained if wl.long_step else bf16_burst) * wl.tc_over_bf16
    tot = T.totals()
    g_n, g_ms = tot["gemm"]
    q_n, q_ms = tot["quant"]
    gemm_tflops = wl.flops() * kernel_steps / (g_ms * 1e-3) / 1e12
    quant_gbs = wl.quant_bytes() * kernel_steps / (q_ms * 1e-3) / 1e9
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": ranks.world,
        "steps": steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.dtype,
        "data": "synthetic (seeded N(0,1) activations with 1% x20 outlier channels, N(0,1/sqrt(K)) weights, "
                "N(0,0.01) f16 bias)",
        "config": run_config(wl, ranks.world),
        "timing": {"l2": "flushed between timed steps (256 MiB write outside the step events)",
                   "launch": "one CUDA graph per step" if graph is not None else "eager launches"},
        "roofline": {"bound": "tensor", "kernel": wl.gemm_kernel,
                     "achieved": round(gemm_tflops, 1), "peak": round(tc_peak, 1), "unit": "TFLOP/s",
                     "frac": round(gemm_tflops / tc_peak, 4),
                     "peak_source": f"{peak_src} bf16 {kind} x {wl.tc_over_bf16} (nominal "
                                    f"{'FP4' if wl.tc_over_bf16 == FP4_OVER_BF16 else 'FP8'}/BF16 ratio)",
                     "traffic": load_traffic(wl.profile_key, wl.profile_kernel),
                     "algorithmic_bytes_per_step": round(wl.gemm_bytes()),
                     "launches_per_step": g_n // kernel_steps, "avg_launch_ms": round(g_ms / g_n, 4)},
        "quant": {"kernel": wl.quant_kernel, "achieved_gbs": round(quant_gbs, 1), "peak_gbs": hbm,
                  "frac": round(quant_gbs / hbm, 4), "peak_source": f"{peak_src} copy",
                  "bytes_per_step": wl.quant_bytes(), "launches_per_step": q_n // kernel_steps,
                  "avg_launch_ms": round(q_ms / q_n, 4)},
        "gpu_launches": wl.launches * steps,
        "clocks": clk.summary(),
    }
    lf = wl.linear_flops()
    per = {}
    for label, (n, ms) in sorted(T.per_label("gemm").items()):
        if label in lf:
            tf = lf[label] * n / (ms * 1e-3) / 1e12
            per[label] = {"launches_per_step": n // kernel_steps, "avg_launch_ms": round(ms / n, 4),
                          "achieved": round(tf, 1), "frac": round(tf / tc_peak, 4)}
    if per:
        out["roofline"]["per_linear"] = per
    if "gelu" in tot:
        n, ms = tot["gelu"]
        out["gelu"] = {"launches_per_step": n // kernel_steps, "avg_launch_ms": round(ms / n, 4)}
    if not args.no_e2e:
        out["e2e"] = run_e2e(args, wl, ranks, dev)
    return out


def run_e2e(args, wl, ranks, dev):
    """Same metric through the public API with host buffers: every step
    copies its X from pinned host memory to the device, runs the layer(s)
    and copies its Y back to pinned host memory, all inside the timed
    region.  Steps are pipelined on three streams (copy in, compute, copy
    out) with two device buffers each way, so that a step's copies overlap
    its neighbours' compute and the PCIe link carries both directions at
    once; events order each buffer's reuse."""
    x_dev, y_ref = wl.e2e_io()
    x_host = torch.empty(x_dev.shape, dtype=x_dev.dtype, pin_memory=True)
    x_host.copy_(x_dev.cpu())
    y_host = [torch.empty(y_ref.shape, dtype=y_ref.dtype, pin_memory=True) for _ in range(2)]
    x_stage = [torch.empty_like(x_dev) for _ in range(2)]
    y_dev = [torch.empty_like(y_ref) for _ in range(2)]
    ws = wl.e2e_workspace(dev)
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    steps = max(3, min(args.steps, 20 if wl.flops() < 1e14 else 3))

    def step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(comp_done[b])          # x_stage[b] no longer read
            x_stage[b].copy_(x_host, non_blocking=True)
            in_done[b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(in_done[b])
            s_comp.wait_event(out_done[b])         # y_dev[b] already copied out
            wl.e2e_step(x_stage[b], y_dev[b], ws)
            comp_done[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            y_host[b].copy_(y_dev[b], non_blocking=True)
            out_done[b].record(s_out)

    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    ranks.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(steps):
        step(i)
    e1.record(s_out)                               # after the last copy out, which follows everything
    torch.cuda.synchronize()
    ms = ranks.max(e0.elapsed_time(e1))
    ranks.barrier()
    value = ranks.world * wl.flops() * steps / (ms * 1e-3) / 1e12
    return {"value": round(value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
            "d2h_bytes_per_step": y_host[0].numel() * y_host[0].element_size(), "steps": steps,
            "ms_per_step": round(ms / steps, 3),
            "overlap": "copy in / compute / copy out on three streams, two device buffers each way"}


def load_traffic(workload, kernel="mxfp8_gemm"):
    """DRAM bytes per GEMM launch from the committed ncu summary
    (profiles/<kernel>_<workload>.json), if it was taken on the kernel's
    current source files; else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.json")
    try:
        d = json.load(open(path))
        from mxfp8_w8a8_quantized_b200 import build
        if d.get("kernel_source_sha") != build.source_sha(kernel):
            return None
        return d["dram_bytes_per_launch"]
    except Exception:
        return None


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(wl, rows):
    """A bounded sample of a single-linear workload for the oracle: `rows`
    rows of X and all of W (quantized by the oracle outside the timed region,
    as weights are offline)."""
    import numpy as np

    import oracle
    from mxfp8_w8a8_quantized_b200 import synth
    x = synth.activations(rows, wl.K, wl.seed, index=100)
    w = synth.weights(wl.N, wl.K, wl.seed, index=100)
    b = synth.bias(wl.N, wl.seed, index=100)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    bb = b.view(torch.int16).numpy().view(np.uint16)
    if wl.scheme == "fp8rowwise":
        wq, ws = oracle.quantize_rowwise_f32(w.numpy())
    elif wl.scheme == "nvfp4":
        wb = w.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        gw = oracle.nvfp4_global_scale(np.abs(w.to(torch.bfloat16).float().numpy()).max())
        gx = oracle.nvfp4_global_scale(np.abs(x.float().numpy()).max())
        wq, ws = oracle.nvfp4_quantize_bf16(wb, gw)
        return xb, (wq, ws, gx, gw), None, bb, wl.scheme
    else:
        wq, ws = oracle.quantize_f32(w.numpy())
    return xb, wq, ws, bb, wl.scheme


def oracle_step(xb, wq, ws, bb, scheme):
    """One step of the oracle on the sample: quantize the rows, FP64 linear."""
    import oracle
    if scheme == "fp8rowwise":
        xq, xs = oracle.quantize_rowwise_bf16(xb)
        return oracle.linear_rowwise(xq, xs, wq, ws, bb)
    if scheme == "nvfp4":
        wq4, ws4, gx, gw = wq
        xq, xs = oracle.nvfp4_quantize_bf16(xb, gx)
        return oracle.nvfp4_linear(xq, xs, gx, wq4, ws4, gw, bb)
    xq, xs = oracle.quantize_bf16(xb)
    return oracle.linear(xq, xs, wq, ws, bb)


def size_sample(wl, target_s, max_rows=None):
    """Rows whose oracle step takes about target_s seconds."""
    rows, dt = 4, 0.0
    for _ in range(6):
        sample = oracle_sample(wl, rows)
        t0 = time.perf_counter()
        oracle_step(*sample)
        dt = time.perf_counter() - t0
        if dt >= 0.5 * target_s:
            break
        rows = int(min(wl.M, max(rows * 2, rows * 0.9 * target_s / max(dt, 1e-3))))
        if max_rows:
            rows = min(rows, max_rows)
    return rows


def chain_oracle_sample(wl):
    """A bounded sample of a chained workload for the oracle: video-token
    rows through the FFN pair, or through one block (its text-token linears
    on a proportional number of text rows, at least one).  Weights are
    quantized by the oracle here, outside any timed region.  Returns
    make(rows) -> (run, flops)."""
    import numpy as np

    import oracle
    from mxfp8_w8a8_quantized_b200 import synth

    def lin(K, N, i):
        wq, ws = oracle.quantize_f32(synth.weights(N, K, wl.seed, index=200 + i).numpy())
        b = synth.bias(N, wl.seed, index=200 + i).view(torch.int16).numpy().view(np.uint16)
        return wq, ws, b

    def apply(x_bits, w):
        xq, xs = oracle.quantize_bf16(x_bits)
        return oracle.bf16_rne(oracle.linear(xq, xs, *w))

    def rows_of(n, K, index):
        return synth.activations(n, K, wl.seed, index=index).view(torch.int16).numpy().view(np.uint16)

    H, F = wl.K, wl.N
    if isinstance(wl, FFNPairWorkload):
        l0, l2 = lin(H, F, 0), lin(F, H, 1)

        def make(rows):
            x = rows_of(rows, H, 300)
            return (lambda: apply(oracle.gelu_tanh_bf16(apply(x, l0)), l2)), 2 * 2.0 * rows * H * F
        return make
    L = {name: lin(K, N, i) for i, (name, K, N, _) in enumerate(synth.block_linears())}

    def make(rows):
        trows = max(1, round(rows * wl.T / wl.M))
        x, ctx = rows_of(rows, H, 300), rows_of(trows, H, 301)

        def run():
            for name in ("attn1.to_q", "attn1.to_k"):
                apply(x, L[name])
            o1 = apply(apply(x, L["attn1.to_v"]), L["attn1.to_out"])
            o2 = apply(apply(o1, L["attn2.to_q"]), L["attn2.to_out"])
            for name in ("attn2.to_k", "attn2.to_v"):
                apply(ctx, L[name])
            return apply(oracle.gelu_tanh_bf16(apply(o2, L["ffn.net.0.proj"])), L["ffn.net.2"])
        return run, 2.0 * (rows * (6 * H * H + 2 * H * F) + trows * 2 * H * H)
    return make


def is_single_linear(wl):
    return type(wl) in (LinearWorkload, FP8RowwiseLinearWorkload, NVFP4LinearWorkload)


def size_chain(wl, target_s):
    """A chained workload's oracle pass on a row sample grown until one pass
    takes about target_s: (rows, run, flops of one pass, seconds of the last
    sizing pass, description)."""
    make = chain_oracle_sample(wl)
    rows = 2
    for _ in range(8):
        run, fl = make(rows)
        t0 = time.perf_counter()
        run()
        dt = time.perf_counter() - t0
        if dt >= 0.5 * target_s or rows >= wl.M:
            break
        rows = int(min(wl.M, max(rows * 2, rows * 0.9 * target_s / max(dt, 1e-3))))
    what = "the FFN pair" if isinstance(wl, FFNPairWorkload) else "one block (text linears on a proportional " \
        "number of text rows)"
    desc = f"{rows} video-token rows through {what}: quantize + FP64 linear per linear, GELU; weights quantized " \
           "outside the timed region"
    return rows, run, fl, dt, desc


def cpu_baseline(wl, target_s):
    import oracle
    if not is_single_linear(wl):
        rows, run, fl, dt, desc = size_chain(wl, target_s)
        return {"value": round(fl / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
                "kind": "oracle", "sample": f"{desc}; {dt:.1f} s"}
    rows = size_sample(wl, target_s)
    sample = oracle_sample(wl, rows)
    t0 = time.perf_counter()
    oracle_step(*sample)
    dt = time.perf_counter() - t0
    return {"value": round(2.0 * rows * wl.N * wl.K / dt / 1e12, 6), "unit": "TFLOP/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{rows} of {wl.M} rows (quantize + FP64 linear over all {wl.N} columns, K={wl.K}); "
                      f"weights quantized outside the timed region; {dt:.1f} s"}


def run_reference(args, ranks):
    """The oracle as the reference arm: CPU, rank 0 only."""
    import oracle
    wl = make_workload(args.workload, scheme=args.scheme)
    if ranks.rank != 0:
        return None
    budget = args.reference_seconds  # warm-up + timed steps together
    n_steps = args.steps + args.warmup
    if is_single_linear(wl):
        rows = size_sample(wl, budget / n_steps)
        data = oracle_sample(wl, rows)
        run, fl = (lambda: oracle_step(*data)), 2.0 * rows * wl.N * wl.K
        sample = f"{rows} of {wl.M} rows per step (quantize + FP64 linear over all {wl.N} columns, K={wl.K})"
    else:
        rows, run, fl, _, desc = size_chain(wl, budget / n_steps)
        sample = f"{desc}, per step"
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = time.perf_counter() - t0
    value = fl * args.steps / dt / 1e12
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 6),
        "unit": "TFLOP/s",
        "n_gpus": ranks.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (same recipe as the GPU arm)",
        "config": run_config(wl, ranks.world),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse(argv)
    if args.impl == "reference":
        # CPU only: rank 0 runs the oracle and prints; other ranks exit at once
        out = run_reference(args, Ranks())
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks(backend="nccl", device=dev)
    try:
        out = run_ours(args, ranks, dev)
        if ranks.rank == 0:
            if ranks.world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline(make_workload(args.workload, scheme=args.scheme),
                                                   args.cpu_seconds)
            print(json.dumps(out), flush=True)
    finally:
        ranks.close()


if __name__ == "__main__":
    main()
