"""Benchmark of the block-scaled linear-layer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

Default workload (N=1): the Wan-2.1-14B-shaped FFN as two NVFP4 W4A4 linear
layers, fc_in A bf16 [32760, 5120] ~N(0,1) x W [13824, 5120]^T ~N(0, 1/sqrt(5120)),
then fc_out A bf16 [32760, 13824] (GELU-shaped) x W [5120, 13824]^T
~N(0, 1/sqrt(13824)); static activation scale 1.0; weights quantized once
before timing (load time).  One step = for each layer, quantize its resident
input (NVFP4 kernel) and run the block-scaled GEMM with alpha fused (tcgen05
kernel); the K timed steps are replayed as one CUDA graph with timing events
recorded as graph nodes around each step (the per-kernel split comes from a
second graph with events between the kernels).  `value` = sum of 2*M*N*K over
the layers per step / step time (TFLOP/s), summed over ranks; L2 is flushed
(256 MiB write) before every timed step, outside the timed events.

Other --config values (wan13, wan14_in, wan14_out, mxfp8, skinny_m<M>,
skinny_out_m<M>, tiny)
time the corresponding one-layer workload the same way; --config loadtime times
the load-time conversion of the 240 weights of a 40-block DiT stack (GB/s).

--impl reference times the CPU oracle (oracle/, plain C + numpy float64) on a
bounded row sample of every layer of the same workload, on the host cores; the
default run's cpu_baseline times the same oracle step.

Under torchrun (N > 1) every rank runs the same workload on its own GPU
(replicas; the path has no exchange step), timing is the max over ranks, and
`value` is the total over ranks (weak scaling).
"""
from __future__ import annotations

import argparse
import contextlib
import ctypes
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 GEMM TFLOP/s & % dense-FP4 peak; quantize GB/s & % HBM (1×B200)"
FP4_PER_BF16 = 4.0  # nominal dense FP4 / BF16 tensor rate (9 / 2.25 PFLOP/s)
FP8_PER_BF16 = 2.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _code_only(src: str) -> str:
    """C/CUDA source without comments and with whitespace runs collapsed, so
    that an edit of comments alone keeps the hash of the kernels."""
    out, i, n = [], 0, len(src)
    while i < n:
        if src.startswith("//", i):
            i = src.find("\n", i)
            i = n if i < 0 else i
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif src[i] == '"':  # string literal: kept as is
            j = i + 1
            while j < n and src[j] != '"':
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(src[i])
            i += 1
    return " ".join("".join(out).split())


# the sources each timed kernel is compiled from (its own file and the shared headers)
KERNEL_SOURCES = {
    "nvfp4_gemm": ("gemm.cu", "bsp_device.cuh", "bsp_internal.h"),
    "mxfp8_gemm": ("gemm.cu", "bsp_device.cuh", "bsp_internal.h"),
    "nvfp4_quantize": ("quantize.cu", "bsp_device.cuh", "bsp_internal.h", "norm_stats.cuh"),
    "nvfp4_rmsnorm_quantize": ("quantize.cu", "bsp_device.cuh", "bsp_internal.h", "norm_stats.cuh"),
    "nvfp4_layernorm_quantize": ("quantize.cu", "bsp_device.cuh", "bsp_internal.h", "norm_stats.cuh"),
    "mxfp8_quantize": ("quantize.cu", "bsp_device.cuh", "bsp_internal.h", "norm_stats.cuh"),
}


def source_hash(files=None) -> str:
    """Identifies kernel sources (by default every csrc/*.cu, *.cuh, *.h;
    comments and layout ignored) that a committed ncu capture was taken on."""
    h = hashlib.sha256()
    cdir = os.path.join(ROOT, "block_scaled_precision_05_b200", "csrc")
    names = sorted(files) if files else sorted(os.listdir(cdir))
    for name in names:
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(cdir, name), encoding="utf-8") as f:
                h.update(name.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def kernel_source_hash(kernel: str) -> str:
    return source_hash(KERNEL_SOURCES.get(kernel))


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time (every rank calls this at the same point)."""
    if world == 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(work_per_rank_step: float, world: int, steps: int, total_ms: float) -> float:
    """Units per second over all ranks: every rank did `steps` steps of the
    same work in (at most) the slowest rank's time."""
    return world * work_per_rank_step * steps / (total_ms * 1e-3)


def traffic_for(kernel: str, workload: str):
    """Per-launch DRAM bytes of `kernel` on `workload` from the committed ncu
    summary, or None when missing or taken on different kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {  # nvmlClocksEventReason bits
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.samples, self.reasons = [], 0
        self.reason_samples = self.reason_errors = self.clock_errors = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            self._ok = False
        self._period = period_s
        self._t = threading.Thread(target=self._run, daemon=True)

    def _handle(self, idx):
        import torch
        nv = self._nv
        try:
            uuid = str(torch.cuda.get_device_properties(idx).uuid)
            return nv.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(idx)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
            except Exception:
                self.clock_errors += 1
            try:
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.reason_samples += 1
            except Exception:
                self.reason_errors += 1
            time.sleep(self._period)

    def __enter__(self):
        if self._ok:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._ok:
            self._t.join()

    def summary(self):
        if not self._ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        unknown = self.reasons & ~sum(self.REASONS)
        if unknown:
            names.append(f"other_bits_{unknown:#x}")
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_min_mhz": min(self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": names, "reason_mask": f"{self.reasons:#x}",
                "samples": len(self.samples), "reason_samples": self.reason_samples,
                "reason_errors": self.reason_errors}


# --------------------------------------------------------------------------- workloads
def make_workloads(name: str, rows: int = 0):
    """[(Linear, kind)] of the layers one step runs, in order (rows > 0: the
    large-M workloads with that many activation rows, for profiler captures)."""
    from block_scaled_precision_05_b200 import workloads as wl
    kw = {"M": rows} if rows > 0 else {}
    if name == "wan14":  # the FFN: fc_in then fc_out, each on its own resident input
        return [(wl.wan14_in(**kw), "nvfp4"), (wl.wan14_out(**kw), "nvfp4")]
    if name == "wan13":
        return [(wl.wan13(**kw), "nvfp4")]
    if name == "tiny":
        return [(wl.tiny(), "nvfp4")]
    if name in ("wan14_in", "wan14_out"):
        return [(getattr(wl, name)(**kw), "nvfp4")]
    if name == "mxfp8":
        return [(wl.mxfp8(**kw), "mxfp8")]
    if name.startswith("skinny_m"):
        return [(wl.skinny(int(name[len("skinny_m"):])), "nvfp4")]
    if name.startswith("skinny_out_m"):
        return [(wl.skinny_out(int(name[len("skinny_out_m"):])), "nvfp4")]
    raise SystemExit(f"unknown --config {name}")


def make_workload(name: str):
    """The single layer of a one-layer configuration."""
    layers = make_workloads(name)
    if len(layers) != 1:
        raise SystemExit(f"--config {name} has {len(layers)} layers")
    return layers[0]


NORM_EPS = 1e-6
WORKLOAD_TITLES = {
    "wan14": "Wan-2.1-14B-shaped FFN, NVFP4 W4A4: fc_in A[32760,5120] x W[13824,5120]^T, then fc_out "
             "A[32760,13824] x W[5120,13824]^T (fc_out input: GELU-shaped, resident)",
}


def norm_gamma(lin):
    """Seeded norm weight for --norm rmsnorm / layernorm: 1 + 0.2 N(0, 1), bf16 bits."""
    from block_scaled_precision_05_b200 import workloads as wl
    rng = np.random.default_rng(77)
    return wl.f32_to_bf16_bits((1.0 + 0.2 * rng.standard_normal(lin.K)).astype(np.float32))


def norm_beta(lin):
    """Seeded LayerNorm bias for --norm layernorm: 0.1 N(0, 1), bf16 bits."""
    from block_scaled_precision_05_b200 import workloads as wl
    rng = np.random.default_rng(78)
    return wl.f32_to_bf16_bits((0.1 * rng.standard_normal(lin.K)).astype(np.float32))


def apply_input_format(lin, kind, fmt):
    """fp16 activations (--input f16, NVFP4 only): the workload's bf16 values
    rounded to fp16 on the host; the oracle quantizes the same fp16 bits."""
    lin.fmt = "bf16"
    if fmt == "f16":
        if kind != "nvfp4":
            raise SystemExit("--input f16 applies to the NVFP4 workloads")
        f32 = (np.ascontiguousarray(lin.A).astype(np.uint32) << 16).view(np.float32)
        lin.A = f32.astype(np.float16).view(np.uint16)
        lin.fmt = "f16"
    return lin


def describe(layers, args):
    """The `config` object of the JSON line; identical in both arms."""
    lines = [f"{lin.name}: {kind.upper()} linear A[{lin.M},{lin.K}] x W[{lin.N},{lin.K}]^T"
             + (" + bias" if lin.bias is not None else "")
             + (" (per-token activation scales)" if lin.per_token else "") for lin, kind in layers]
    d = {"workload": WORKLOAD_TITLES.get(args.config, "; ".join(lines))}
    if len(layers) > 1:
        d["layers"] = lines
    lin0, kind0 = layers[0]
    if len(layers) == 1:
        d.update({"M": lin0.M, "N": lin0.N, "K": lin0.K})
    d["flop_per_step"] = int(sum(lin.flops for lin, _ in layers))
    d["l2"] = "flushed before every timed step (256 MiB write, outside the timed events)"
    d["parallelism"] = "replicas (one process per GPU, no exchange)"
    d["activation_dtype"] = "fp16" if args.input == "f16" else "bf16"
    if kind0 == "nvfp4":
        d["activation_sf_layout"] = args.sf_layout
        d["weight_global_scale"] = "256*6/amax (4over6)" if args.four_over_six else "448*6/amax"
    if args.norm == "rmsnorm":
        d["producer"] = f"RMSNorm (gamma 1+0.2N(0,1), eps {NORM_EPS:g}) fused into the quantizer"
    elif args.norm == "layernorm":
        d["producer"] = (f"LayerNorm (gamma 1+0.2N(0,1), beta 0.1N(0,1), eps {NORM_EPS:g}) fused into the "
                         "quantizer")
    return d


def quant_bytes(M, K, kind, sf_layout="128x4"):
    """Algorithmic HBM bytes of one activation quantize launch."""
    if kind == "nvfp4":
        row_tile = 8 if sf_layout == "8x4" else 128
        return M * K * 2 + M * K // 2 + (-(-M // row_tile) * row_tile) * (-(-(K // 16) // 4) * 4)
    return M * K * 2 + M * K + (-(-M // 128) * 128) * (-(-(K // 32) // 4) * 4)


def skinny_gemm_bytes(M, N, K, kind):
    """Algorithmic HBM bytes of a GEMM that streams the weight once (M <= 128):
    operand codes, their scales and the bf16 output."""
    c, g = (0.5, 16) if kind == "nvfp4" else (1.0, 32)
    return int((M * K + N * K) * c + (M + N) * (K // g) + 2 * M * N)


def quant_kernel_name(kind, norm):
    return {"rmsnorm": "nvfp4_rmsnorm_quantize", "layernorm": "nvfp4_layernorm_quantize"}.get(norm,
                                                                                              f"{kind}_quantize")


def roofline_of(parts, peaks, peak_src, traffic):
    """Roofline of the dominant kernel.  `parts` lists per layer (lin, kind,
    q_ms, g_ms, q_bytes); the kernel with the most time over the step is the
    dominant one, and for several layers its figures are the step's totals
    (achieved = work over all its launches / their summed duration, traffic =
    mean per launch)."""
    q_tot = sum(p[2] for p in parts)
    g_tot = sum(p[3] for p in parts)
    kind = parts[0][1]
    if all(p[0].M <= 128 for p in parts):
        gb = sum(skinny_gemm_bytes(p[0].M, p[0].N, p[0].K, p[1]) for p in parts)
        a = gb / (g_tot * 1e-3) / 1e9
        return {"kernel": f"{kind}_gemm", "bound": "hbm", "achieved": round(a, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(a / peaks["hbm_gbs"], 4), "traffic": traffic("gemm"),
                "peak_source": f"{peak_src}: hbm_gbs",
                "algorithmic": f"{gb // len(parts)} bytes per launch (operand codes + scales + output)"}
    if g_tot >= q_tot:
        ratio = FP4_PER_BF16 if kind == "nvfp4" else FP8_PER_BF16
        peak = peaks["bf16_tflops"] * ratio
        flops = sum(p[0].flops for p in parts)
        a = flops / (g_tot * 1e-3) / 1e12
        per = "; ".join(f"{p[0].name} {p[0].flops:.4g}" for p in parts)
        return {"kernel": f"{kind}_gemm", "bound": "tensor", "achieved": round(a, 1), "peak": round(peak, 1),
                "unit": "TFLOP/s", "frac": round(a / peak, 4), "traffic": traffic("gemm"),
                "peak_source": f"{peak_src}: bf16_tflops (burst) x {ratio:g} nominal {kind} ratio",
                "algorithmic": f"2*M*N*K flop per launch ({per})"}
    qb = sum(p[4] for p in parts)
    a = qb / (q_tot * 1e-3) / 1e9
    return {"kernel": "quantize", "bound": "hbm", "achieved": round(a, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(a / peaks["hbm_gbs"], 4), "traffic": traffic("quantize"),
            "peak_source": f"{peak_src}: hbm_gbs", "algorithmic": f"{qb // len(parts)} bytes per launch"}


# --------------------------------------------------------------------------- our arm
class LayerRun:
    """One layer of the timed step on the device: its resident input, the
    weight quantized at load time, preallocated outputs, and the two launches."""

    def __init__(self, lin, kind, args, dev):
        import torch

        from block_scaled_precision_05_b200 import api
        self.api, self.lin, self.kind, self.args, self.dev = api, lin, kind, args, dev
        self.a_dtype = torch.float16 if lin.fmt == "f16" else torch.bfloat16
        self.A = self.up(lin.A, self.a_dtype)
        self.gamma = self.beta = None
        if args.norm != "none":
            if kind != "nvfp4" or lin.fmt != "bf16":
                raise SystemExit(f"--norm {args.norm} applies to the bf16 NVFP4 workloads")
            self.gamma = self.up(norm_gamma(lin))
            if args.norm == "layernorm":
                self.beta = self.up(norm_beta(lin))
        W = self.up(lin.W)
        bias = None if lin.bias is None else self.up(lin.bias)
        if kind == "nvfp4":
            self.layer = api.NVFP4Linear(W, bias, per_token=lin.per_token, four_over_six=args.four_over_six)
        else:
            self.layer = api.MXFP8Linear(W, bias)
        del W
        M, K = lin.M, lin.K
        if kind == "nvfp4" and args.sf_layout == "8x4" and (M > 64 or args.norm != "none"):
            raise SystemExit("--sf-layout 8x4 applies to NVFP4 workloads with M <= 64 and no fused norm")
        self.xq = self.new_xq()
        self.D = torch.empty((M, lin.N), dtype=torch.bfloat16, device=dev)
        self.qname = quant_kernel_name(kind, args.norm)

    def up(self, a, dtype=None):
        import torch
        dtype = dtype or torch.bfloat16
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(dtype).to(self.dev)

    def new_xq(self):
        import torch
        api, lin, M, K = self.api, self.lin, self.lin.M, self.lin.K
        if self.kind == "nvfp4":
            xq = api.NVFP4Tensor(torch.empty((M, K // 2), dtype=torch.uint8, device=self.dev),
                                 torch.empty(api.nvfp4_sf_bytes(M, K, self.args.sf_layout), dtype=torch.uint8,
                                             device=self.dev), K, sf_layout=self.args.sf_layout)
            if lin.per_token:
                xq.row_gs = torch.empty(M, dtype=torch.float32, device=self.dev)
                xq.row_inv_gs = torch.empty(M, dtype=torch.float32, device=self.dev)
            return xq
        return api.MXFP8Tensor(torch.empty((M, K), dtype=torch.uint8, device=self.dev),
                               torch.empty(api.mxfp8_sf_bytes(M, K), dtype=torch.uint8, device=self.dev), K)

    def quantize(self, x=None, out=None):
        api, args, lin, layer = self.api, self.args, self.lin, self.layer
        x = self.A if x is None else x
        out = self.xq if out is None else out
        gs = None if lin.per_token else getattr(layer, "gs_x", None)
        if args.norm == "rmsnorm":
            api.nvfp4_rmsnorm_quantize(x, self.gamma, NORM_EPS, gs, per_row=lin.per_token, out=out)
        elif args.norm == "layernorm":
            api.nvfp4_layernorm_quantize(x, self.gamma, self.beta, NORM_EPS, gs, per_row=lin.per_token, out=out)
        elif self.kind == "nvfp4":
            api.nvfp4_quantize(x, gs, per_row=lin.per_token, out=out, sf_layout=args.sf_layout)
        else:
            api.mxfp8_quantize(x, out=out)

    def gemm(self, a=None, b=None, out=None):
        api, layer = self.api, self.layer
        a = self.xq if a is None else a
        b = layer.weight if b is None else b
        out = self.D if out is None else out
        if self.kind == "nvfp4":
            api.nvfp4_gemm(a, b, layer.alpha, a.row_inv_gs if self.lin.per_token else None, layer.bias, out=out)
        else:
            api.mxfp8_gemm(a, b, None, layer.bias, out=out)

    def call(self, x):
        """The public layer call (e2e): quantize (or norm + quantize) and GEMM."""
        layer, args = self.layer, self.args
        if args.norm == "rmsnorm":
            return layer(x, pre_quantized=layer.rmsnorm_quantize_input(x, self.gamma, NORM_EPS))
        if args.norm == "layernorm":
            return layer(x, pre_quantized=layer.layernorm_quantize_input(x, self.gamma, self.beta, NORM_EPS))
        if self.kind == "nvfp4":
            return layer(x, sf_layout=args.sf_layout)
        return layer(x)

    @property
    def w_bytes(self):
        w = self.layer.weight
        return (w.codes.numel() if self.kind == "nvfp4" else w.q.numel()) + w.sf.numel()

    @property
    def a_bytes(self):
        x = self.xq
        return (x.codes.numel() if self.kind == "nvfp4" else x.q.numel()) + x.sf.numel()

    def clone_xq(self):
        import torch
        x = self.xq
        if self.kind == "nvfp4":
            t = self.api.NVFP4Tensor(torch.empty_like(x.codes), torch.empty_like(x.sf), self.lin.K,
                                     sf_layout=x.sf_layout)
            if self.lin.per_token:
                t.row_gs, t.row_inv_gs = torch.empty_like(x.row_gs), torch.empty_like(x.row_inv_gs)
            return t
        return self.api.MXFP8Tensor(torch.empty_like(x.q), torch.empty_like(x.sf), self.lin.K)

    def clone_weight(self):
        w, K = self.layer.weight, self.lin.K
        if self.kind == "nvfp4":
            return self.api.NVFP4Tensor(w.codes.clone(), w.sf.clone(), K)
        return self.api.MXFP8Tensor(w.q.clone(), w.sf.clone(), K)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from block_scaled_precision_05_b200 import api

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    specs = [(apply_input_format(lin, kind, args.input), kind) for lin, kind in make_workloads(args.config, args.rows)]
    runs = [LayerRun(lin, kind, args, dev) for lin, kind in specs]
    flops = float(sum(r.lin.flops for r in runs))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    if args.profile_launches:
        # a short eager run for a profiler capture: set-up, then N steps
        for _ in range(args.profile_launches):
            for r in runs:
                r.quantize()
                r.gemm()
        torch.cuda.synchronize()
        if api.device_status() != 0:
            raise RuntimeError("device error word set")
        return {"profile_launches": args.profile_launches, "config": args.config,
                "layers": [r.lin.name for r in runs]}

    for _ in range(args.warmup):
        flush.zero_()
        for r in runs:
            r.quantize()
            r.gemm()
    torch.cuda.synchronize()
    if api.device_status() != 0:
        raise RuntimeError("device error word set during warm-up")

    # The timed region is one CUDA graph holding all K steps back to back: per
    # step an L2 flush, then a timing event, every layer's quantize and GEMM
    # launches and a second timing event (events are graph nodes; no Python or
    # ctypes launch latency inside the measured intervals).  The library is
    # capturable (no allocation, no host synchronisation).  A second graph of
    # the same steps with an event also between every two kernels gives the
    # per-kernel split; every event interval on this device carries a launch
    # floor of about 6 us (an empty kernel between two event nodes reads 6.1 us).
    nk = 2 * len(runs)

    def step(evs, split):  # records on the current (capturing) stream
        flush.zero_()
        evs[0].record()
        for i, r in enumerate(runs):
            r.quantize()
            if split:
                evs[2 * i + 1].record()
            r.gemm()
            if split or i == len(runs) - 1:
                evs[2 * i + 2].record()

    def graph_of(steps, split):
        evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(nk + 1)] for _ in range(steps)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for s in range(steps):
                step(evs[s], split)
        return g, evs

    g_warm, ev_warm = graph_of(1, False)  # the events must outlive the graph that records them
    for _ in range(args.warmup):
        g_warm.replay()
    g_timed, ev = graph_of(args.steps, False)
    g_split, ev_split = graph_of(args.steps, True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier(device_ids=[local_rank])
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        g_timed.replay()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier(device_ids=[local_rank])
    g_split.replay()  # untimed for the step value: per-kernel durations only
    torch.cuda.synchronize()
    step_ms = [ev[s][0].elapsed_time(ev[s][nk]) for s in range(args.steps)]
    split_ms = [[statistics.mean(ev_split[s][j].elapsed_time(ev_split[s][j + 1]) for s in range(args.steps))
                 for j in range(nk)]]
    split_ms = split_ms[0]
    total_ms = max_over_ranks(float(sum(step_ms)), world, dev)
    if api.device_status() != 0:
        raise RuntimeError("device error word set during timing")
    ms_per_step = total_ms / args.steps
    value = whole_job_rate(flops, world, args.steps, total_ms) / 1e12
    del g_warm, g_timed, g_split, ev_warm

    # ---- per-kernel durations for the roofline: R launches of one kernel back to
    # back in a CUDA graph between two events, rotating through enough distinct
    # operand buffers (> 3x L2 in total) that every launch reads its streamed
    # operand from DRAM.  Back to back, consecutive launches hide each other's
    # launch latency as they do in a model; the per-step split above carries an
    # event-interval floor of about 6 us per kernel and is reported beside it.
    # R launches last about 2 ms in all (4 to 24), short enough to stay a burst
    # like the timed steps rather than a sustained power-capped loop.
    def launches_for(ms):
        return int(min(24, max(4, 2.0 / max(ms, 1e-3))))

    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size

    def rotations(streamed_bytes):
        return int(min(8, max(2, -(-3 * l2_bytes // max(1, streamed_bytes)))))

    def back_to_back(launch, n_rot, R):
        for i in range(n_rot):
            launch(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(R):
                launch(i % n_rot)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g.replay()
        torch.cuda.synchronize()
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) / R

    b2b = []  # per layer: (quantize ms, GEMM ms, R_q, R_g)
    for i, r in enumerate(runs):
        # the GEMM streams A (large M) or the weight (skinny M) from DRAM
        rotate_weight = r.w_bytes > r.a_bytes
        nq = rotations(r.A.numel() * r.A.element_size())
        nx = max(nq, 1 if rotate_weight else rotations(r.a_bytes))
        A_rot = [r.A] + [r.A.clone() for _ in range(nq - 1)]
        xq_rot = [r.xq] + [r.clone_xq() for _ in range(nx - 1)]
        R_q, R_g = launches_for(split_ms[2 * i]), launches_for(split_ms[2 * i + 1])
        q_ms = back_to_back(lambda j: r.quantize(A_rot[j % nq], xq_rot[j]), nx, max(R_q, nx))
        ng = rotations(max(r.w_bytes, r.a_bytes))
        w_rot = [r.layer.weight] + [r.clone_weight() for _ in range(ng - 1)] if rotate_weight else None
        D_rot = [r.D] + [torch.empty_like(r.D) for _ in range(min(ng, 2) - 1)]

        def gemm_launch(j):
            a = r.xq if rotate_weight else xq_rot[j]
            b = w_rot[j] if rotate_weight else None
            r.gemm(a, b, D_rot[j % len(D_rot)])

        g_ms = back_to_back(gemm_launch, ng if rotate_weight else nx, R_g)
        del A_rot, xq_rot, D_rot, w_rot
        torch.cuda.empty_cache()
        b2b.append((max_over_ranks(q_ms, world, dev), max_over_ranks(g_ms, world, dev), R_q, R_g))

    # ---- end to end through the public API: every step copies each layer's
    # input from pinned host memory and its result back to pinned host memory.
    # With large copies the steps are pipelined as a serving loop would run
    # them: the copy-in of step i+1 and the copy-out of step i-1 run on their
    # own streams while step i computes (two device input buffers and two host
    # output buffers per layer).  With small copies (skinny M) the extra stream
    # bookkeeping costs more host time than it hides, and the steps run on one
    # stream.
    A_host = [torch.from_numpy(np.ascontiguousarray(r.lin.A).view(np.int16)).view(r.a_dtype).pin_memory()
              for r in runs]
    D_host = [[torch.empty((r.lin.M, r.lin.N), dtype=torch.bfloat16).pin_memory() for _ in range(2)] for r in runs]
    A_dev = [[torch.empty_like(r.A) for _ in range(2)] for r in runs]
    e2e_steps = max(2, min(args.steps, 20))
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    h2d = sum(a.numel() * a.element_size() for a in A_host)
    d2h = sum(d[0].numel() * 2 for d in D_host)
    pipelined = h2d + d2h > (16 << 20)

    def e2e_step(i):
        b = i % 2
        if not pipelined:
            for li, r in enumerate(runs):
                A_dev[li][0].copy_(A_host[li], non_blocking=True)
                D_host[li][0].copy_(r.call(A_dev[li][0]), non_blocking=True)
            return
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_comp[b])  # step i-2 has finished reading A_dev[.][b]
            for li in range(len(runs)):
                A_dev[li][b].copy_(A_host[li], non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        ys = [r.call(A_dev[li][b]) for li, r in enumerate(runs)]
        ev_comp[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            for li, y in enumerate(ys):
                D_host[li][b].copy_(y, non_blocking=True)  # in order after step i-2's copy of D_host[.][b]
                y.record_stream(s_out)

    def e2e_run(n):
        e0, e1, e_out = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
                         torch.cuda.Event())
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(n):
            e2e_step(i)
        e_out.record(s_out)
        stream.wait_event(e_out)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    e2e_run(2)
    if world > 1:
        dist.barrier(device_ids=[local_rank])
    # three runs of e2e_steps steps, the median reported: a single stall of the
    # host (another process, paging of the pinned buffers) lands in one run
    e2e_runs = [e2e_run(e2e_steps) / e2e_steps for _ in range(3)]
    e2e_ms = max_over_ranks(statistics.median(e2e_runs), world, dev)

    # ---- roofline of the dominant kernel
    peaks, peak_src = load_peaks()
    parts = [(r.lin, r.kind, q, g, quant_bytes(r.lin.M, r.lin.K, r.kind, args.sf_layout))
             for r, (q, g, _, _) in zip(runs, b2b)]
    wsuffix = {"rmsnorm": "_rmsnorm", "layernorm": "_layernorm"}.get(args.norm, "")

    def traffic(which):
        vals = [traffic_for(f"{r.kind}_gemm" if which == "gemm" else r.qname, r.lin.name + wsuffix) for r in runs]
        return None if any(v is None for v in vals) else int(sum(vals) / len(vals))

    roof = roofline_of(parts, peaks, peak_src, traffic)
    if roof["kernel"] == "quantize":
        roof["kernel"] = runs[0].qname
    hbm_peak = peaks["hbm_gbs"]
    kernels = {}
    for i, (r, (q_ms, g_ms, R_q, R_g)) in enumerate(zip(runs, b2b)):
        ratio = FP4_PER_BF16 if r.kind == "nvfp4" else FP8_PER_BF16
        tensor_peak = peaks["bf16_tflops"] * ratio
        qb = parts[i][4]
        g_tflops = r.lin.flops / (g_ms * 1e-3) / 1e12
        entry = {r.qname: {"ms": round(q_ms, 5), "GB/s": round(qb / (q_ms * 1e-3) / 1e9, 1),
                           "frac_hbm": round(qb / (q_ms * 1e-3) / 1e9 / hbm_peak, 4)},
                 f"{r.kind}_gemm": {"ms": round(g_ms, 5), "TFLOP/s": round(g_tflops, 1),
                                    "frac_tensor_peak": round(g_tflops / tensor_peak, 4)},
                 "launches_back_to_back": [R_q, R_g],
                 "per_step_event_split_ms": [round(split_ms[2 * i], 5), round(split_ms[2 * i + 1], 5)]}
        if r.lin.M <= 128:
            gb = skinny_gemm_bytes(r.lin.M, r.lin.N, r.lin.K, r.kind)
            entry[f"{r.kind}_gemm"]["frac_hbm"] = round(gb / (g_ms * 1e-3) / 1e9 / hbm_peak, 4)
        kernels[r.lin.name] = entry
    kernels["timing"] = ("each kernel launched R times back to back in one CUDA graph between two events (about "
                         "2 ms), operands rotated through buffers totalling > 3x L2 so each launch streams from "
                         "DRAM; per_step_event_split_ms: events around each kernel inside the timed steps, each "
                         "interval carrying a ~6 us event/launch floor")
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4" if runs[0].kind == "nvfp4" else "mxfp8",
        "data": "synthetic (seeded numpy)", "config": describe(specs, args), "roofline": roof,
        "kernels": kernels,
        "e2e": {"value": round(whole_job_rate(flops, world, 1, e2e_ms) / 1e12, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "ms_per_step": round(e2e_ms, 4), "runs_ms_per_step": [round(v, 4) for v in e2e_runs],
                "steps_per_run": e2e_steps,
                "pipelining": ("each step's copy-in, compute and copy-out on three streams; consecutive steps "
                               "overlap") if pipelined else "none (one stream; small copies)"},
        "gpu_launches": nk * args.steps,
        "timing": ("K steps in one CUDA graph, CUDA events as graph nodes around each step's kernels; L2 flushed "
                   "before every step outside the events"),
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = oracle_baseline(specs, args)
    return out


# --------------------------------------------------------------------------- load-time sweep
def run_loadtime(args, rank, world, local_rank):
    """Load-time weight conversion of a synthetic 14B-class DiT stack: for each
    of the 240 linears of 40 blocks (q, k, v, out 5120x5120; fc_in 13824x5120;
    fc_out 5120x13824; bf16 ~N(0, 0.02), drawn on the device from seeded
    generators), amax -> gs_w = 2688/amax -> NVFP4 quantize: all 240 in one
    nvfp4_quantize_weights launch.  The whole sweep is one CUDA graph; one step
    = one sweep.  The weights (19.7 GB) are far larger than L2.  The same sweep
    as one nvfp4_quantize_weight launch per weight, and as three launches per
    weight (amax, global scale, quantize, plus the amax reset), is timed beside
    it."""
    import torch
    import torch.distributed as dist

    from block_scaled_precision_05_b200 import api
    from block_scaled_precision_05_b200 import workloads as wl

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    shapes = wl.dit_weight_shapes(args.blocks)
    weights, outs, scales = [], [], []
    for i, (b, name, N, K) in enumerate(shapes):
        w = wl.device_weight(b, i % 6, N, K, dev)
        weights.append(w)
        outs.append(api.NVFP4Tensor(torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                                    torch.empty(api.nvfp4_sf_bytes(N, K), dtype=torch.uint8, device=dev), K))
        scales.append(tuple(torch.empty(1, dtype=torch.float32, device=dev) for _ in range(3)))
    from block_scaled_precision_05_b200 import _native as nat
    L = nat.lib()
    ws = api._weight_workspace(dev, nat.BSP_IN_BF16)
    chunks = [list(range(c, min(c + nat.BSP_WEIGHT_BATCH_MAX, len(shapes))))
              for c in range(0, len(shapes), nat.BSP_WEIGHT_BATCH_MAX)]
    descs = []
    for idx in chunks:
        arr = (nat.BspWeightDesc * len(idx))()
        for d, i in zip(arr, idx):
            w, o, (amax, gs, inv) = weights[i], outs[i], scales[i]
            d.w, d.N, d.K, d.ld_w = w.data_ptr(), w.shape[0], w.shape[1], w.shape[1]
            d.amax, d.gs, d.inv_gs, d.codes, d.sf = amax.data_ptr(), gs.data_ptr(), inv.data_ptr(), \
                o.codes.data_ptr(), o.sf.data_ptr()
        descs.append(arr)

    def sweep():
        st = torch.cuda.current_stream().cuda_stream
        for arr in descs:
            nat.check(L.nvfp4_quantize_weights(ctypes.addressof(arr), len(arr), nat.BSP_IN_BF16, api.FP8_FP4_MAX,
                                               ws.data_ptr(), ws.numel(), st), "quantize_weights")

    def sweep_per_weight():
        st = torch.cuda.current_stream().cuda_stream
        for w, o, (amax, gs, inv) in zip(weights, outs, scales):
            N, K = w.shape
            nat.check(L.nvfp4_quantize_weight(w.data_ptr(), nat.BSP_IN_BF16, N, K, K, api.FP8_FP4_MAX,
                                              amax.data_ptr(), gs.data_ptr(), inv.data_ptr(), o.codes.data_ptr(),
                                              o.sf.data_ptr(), ws.data_ptr(), ws.numel(), st), "quantize_weight")

    def sweep_unfused():
        st = torch.cuda.current_stream().cuda_stream
        for w, o, (amax, gs, inv) in zip(weights, outs, scales):
            nat.check(L.bsp_amax_bf16(w.data_ptr(), w.numel(), amax.data_ptr(), st), "amax")
            nat.check(L.bsp_nvfp4_global_scale(amax.data_ptr(), gs.data_ptr(), inv.data_ptr(), st), "gs")
            api.nvfp4_quantize(w, gs, out=o)

    def timed(fn, steps, clocks=None):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        for _ in range(args.warmup):
            g.replay()
        torch.cuda.synchronize()
        if api.device_status() != 0:
            raise RuntimeError("device error word set")
        stream = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier(device_ids=[local_rank])
        torch.cuda.synchronize()
        with (clocks if clocks is not None else contextlib.nullcontext()):
            e0.record(stream)
            for _ in range(steps):
                g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
        del g
        if api.device_status() != 0:
            raise RuntimeError("device error word set")
        return max_over_ranks(e0.elapsed_time(e1), world, dev)

    clocks = ClockSampler(local_rank)
    total_ms = timed(sweep, args.steps, clocks)
    k2 = max(1, args.steps // 2)
    per_weight_ms = timed(sweep_per_weight, k2) / k2
    unfused_ms = timed(sweep_unfused, k2) / k2
    elems = sum(N * K for (_, _, N, K) in shapes)
    # algorithmic bytes of the two passes the conversion needs (the amax pass and
    # the quantize pass, 2 + 2.5625 B/elt); the one-kernel form re-reads a weight
    # from L2 where it fits, which this count does not credit
    nbytes = sum(2 * N * K + 2 * N * K + N * K // 2 + api.nvfp4_sf_bytes(N, K) for (_, _, N, K) in shapes)
    gbs = whole_job_rate(nbytes, world, args.steps, total_ms) / 1e9
    peaks, src = load_peaks()
    return {
        "metric": "load-time NVFP4 weight conversion (amax + global scale + quantize) GB/s", "value": round(gbs, 1),
        "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic (seeded torch, on device)",
        "config": {"workload": f"loadtime: {len(shapes)} DiT linears ({args.blocks} blocks), {elems / 1e9:.2f} G "
                               "bf16 elements", "l2": "inputs (19.7 GB at 40 blocks) far larger than L2",
                   "kernel": "nvfp4_quantize_weights: one cooperative launch for all weights (per weight: amax, "
                             "grid barrier, global scale, quantize last row first)"},
        "roofline": {"kernel": "nvfp4_quantize_weights (whole sweep)", "bound": "hbm", "achieved": round(gbs / world, 1),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(gbs / world / peaks["hbm_gbs"], 4),
                     "traffic": None, "peak_source": f"{src}: hbm_gbs",
                     "algorithmic": f"{nbytes} bytes per sweep (amax pass 2 B/elt; quantize pass 2 B/elt read + "
                                    "0.5 B/elt codes + scales)"},
        "one_launch_per_weight": {"ms_per_step": round(per_weight_ms, 4),
                                  "GB/s_same_bytes": round(nbytes / (per_weight_ms * 1e-3) / 1e9, 1)},
        "unfused": {"ms_per_step": round(unfused_ms, 4),
                    "GB/s_same_bytes": round(nbytes / (unfused_ms * 1e-3) / 1e9, 1),
                    "launches_per_weight": "memset + amax + global scale + quantize"},
        "gpu_launches": len(chunks) * args.steps,
        "clocks": clocks.summary(),
    }


# --------------------------------------------------------------------------- oracle arm
def oracle_step(lin, kind, rows, wq, norm=None):
    """The oracle's linear layer on `rows` of A: (norm,) quantize, decode,
    float64 GEMM, epilogue, bf16 rounding."""
    import oracle
    K = lin.K
    A = lin.A[rows]
    if kind == "nvfp4":
        gs_w, codes_b, sf_b, decB = wq
        fmt = getattr(lin, "fmt", "bf16")
        if norm == "rmsnorm":
            A = oracle.rmsnorm_bf16(A, norm_gamma(lin), oracle.rmsnorm_rstd(A, NORM_EPS))
        elif norm == "layernorm":
            mean, rstd = oracle.layernorm_stats(A, NORM_EPS)
            A = oracle.layernorm_bf16(A, norm_gamma(lin), norm_beta(lin), mean, rstd)
        if lin.per_token:
            gs, inv = oracle.row_global_scales(A, fmt=fmt)
            ca, sa = oracle.nvfp4_quantize(A, gs, per_row=True, fmt=fmt)
            alpha, rs = np.float32(1) / gs_w, inv
        else:
            ca, sa = oracle.nvfp4_quantize(A, 1.0, fmt=fmt)
            alpha, rs = np.float32(1) / (np.float32(1) * gs_w), None
        decA = oracle.nvfp4_dequantize(ca, sa, K)
    else:
        _, _, _, decB = wq
        qa, sa = oracle.mxfp8_quantize(A)
        decA = oracle.mxfp8_dequantize(qa, sa, K)
        alpha, rs = 1.0, None
    y, _ = oracle.linear_reference(decA, decB, alpha=alpha, row_scale=rs, bias=lin.bias)
    return oracle.bf16_round(y)


def oracle_weights(lin, kind, four_over_six=False):
    import oracle
    if kind == "nvfp4":
        gs_w = oracle.nvfp4_global_scale(oracle.amax_bf16(lin.W), 1536.0 if four_over_six else 2688.0)
        cb, sb = oracle.nvfp4_quantize(lin.W, gs_w)
        return gs_w, cb, sb, oracle.nvfp4_dequantize(cb, sb, lin.K)
    qb, sb = oracle.mxfp8_quantize(lin.W)
    return None, qb, sb, oracle.mxfp8_dequantize(qb, sb, lin.K)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def oracle_rows(args, M):
    """Rows of A per layer that one oracle step processes: --ref-rows, or by
    default up to 128 (about a second of oracle work per Wan-14B layer)."""
    if args.ref_rows:
        return min(M, args.ref_rows)
    return M if M <= 128 else 128


class OracleRunner:
    """The oracle's step over the same layers as the GPU step: each step takes
    a fresh random sample of rows of every layer's A (seeded) and runs the whole
    path on them.  Used, unchanged, by the reference arm and by cpu_baseline,
    so both report the same work per step."""

    def __init__(self, specs, args, seed=7):
        self.specs, self.args = specs, args
        self.wq = [oracle_weights(lin, kind, args.four_over_six) for lin, kind in specs]
        self.n = [oracle_rows(args, lin.M) for lin, _ in specs]
        self.rng = np.random.default_rng(seed)
        self.flops = 2.0 * sum(n * lin.N * lin.K for n, (lin, _) in zip(self.n, specs))

    def step(self):
        for (lin, kind), wq, n in zip(self.specs, self.wq, self.n):
            rows = np.sort(self.rng.choice(lin.M, size=n, replace=False))
            oracle_step(lin, kind, rows, wq, self.args.norm)

    def sample(self):
        parts = [f"{n} random rows of {lin.name} A (of {lin.M})" for n, (lin, _) in zip(self.n, self.specs)]
        return ("per step " + ", ".join(parts) + ": quantize + decode + float64 GEMM + epilogue + bf16 rounding; "
                "weights quantized beforehand (load time); plain C + numpy oracle")

    def timed(self, steps, warmup):
        for _ in range(warmup):
            self.step()
        t0 = time.perf_counter()
        for _ in range(steps):
            self.step()
        return time.perf_counter() - t0


def oracle_baseline(specs, args):
    """cpu_baseline: the reference arm's oracle step, timed for about
    --cpu-budget seconds (at least one step after one warm-up step)."""
    orc = OracleRunner(specs, args)
    t1 = orc.timed(1, 1)
    steps = int(max(1, min(50, args.cpu_budget / max(t1, 1e-3))))
    dt = t1 + (orc.timed(steps - 1, 0) if steps > 1 else 0.0)
    return {"value": round(orc.flops * steps / dt / 1e12, 6), "unit": "TFLOP/s",
            "cores": max(os.cpu_count() or 1, blas_threads()), "kind": "oracle", "steps": steps,
            "seconds": round(dt, 2), "sample": orc.sample()}


def run_reference_loadtime(args):
    """The oracle's weight conversion (amax, global scale, quantize) on a bounded
    sample: one 5120x5120 N(0, 0.02) weight per step, drawn with numpy."""
    import oracle
    from block_scaled_precision_05_b200 import workloads as wl
    rng = np.random.default_rng(6)
    N = K = wl.DIT_HIDDEN
    w = wl.normal_bf16(rng, (N, K), 0.02)

    def step():
        gs = oracle.nvfp4_global_scale(oracle.amax_bf16(w))
        oracle.nvfp4_quantize(w, gs)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    nbytes = 4 * N * K + N * K // 2 + oracle.sf_bytes(N, K // 16)  # amax pass + quantize pass, as the GPU arm
    value = nbytes * args.steps / dt / 1e9
    cores = os.cpu_count() or 1
    sample = "one 5120x5120 bf16 weight per step: amax + global scale + NVFP4 quantize (plain C oracle)"
    return {"impl": "reference", "metric": "load-time NVFP4 weight conversion (amax + global scale + quantize) GB/s",
            "value": round(value, 3), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32 (oracle)", "data": "synthetic (seeded numpy)",
            "config": {"workload": f"loadtime: {args.blocks}-block DiT weight conversion (oracle sample)"},
            "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_reference(args):
    """The oracle on the host cores as the reference arm: the same layers, a
    bounded row sample of each per step (the same runner as cpu_baseline)."""
    if args.config == "loadtime":
        return run_reference_loadtime(args)
    specs = [(apply_input_format(lin, kind, args.input), kind) for lin, kind in make_workloads(args.config)]
    orc = OracleRunner(specs, args)
    dt = orc.timed(args.steps, args.warmup)
    value = orc.flops * args.steps / dt / 1e12
    cores = max(os.cpu_count() or 1, blas_threads())
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64 (oracle)", "data": "synthetic (seeded numpy)", "config": describe(specs, args),
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": orc.sample()},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# --------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="wan14")
    ap.add_argument("--sf-layout", choices=["128x4", "8x4"], default="128x4",
                    help="activation scale layout of the NVFP4 workloads (8x4: M <= 64)")
    ap.add_argument("--norm", choices=["none", "rmsnorm", "layernorm"], default="none",
                    help="NVFP4 workloads: fuse a norm of the activation into the quantizer")
    ap.add_argument("--input", choices=["bf16", "f16"], default="bf16",
                    help="activation dtype of the NVFP4 workloads (f16: the bf16 values rounded to fp16)")
    ap.add_argument("--four-over-six", action="store_true",
                    help="NVFP4 weight global scale 256*6/amax (the 4over6 setting) instead of 448*6/amax")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-rows", type=int, default=0,
                    help="rows of each layer's A per oracle step (reference arm and cpu_baseline; 0: up to 128)")
    ap.add_argument("--profile-launches", type=int, default=0,
                    help="set up, run this many untimed eager steps and exit (for a profiler capture)")
    ap.add_argument("--rows", type=int, default=0,
                    help="with --profile-launches: activation rows of the large-M workloads (0: the config's)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--blocks", type=int, default=40, help="DiT blocks for --config loadtime")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.rows and not args.profile_launches:
        ap.error("--rows applies to --profile-launches runs only")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0

    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        out = (run_loadtime if args.config == "loadtime" else run_ours)(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
