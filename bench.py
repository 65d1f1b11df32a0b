"""Benchmark of the block-scaled linear-layer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

Default workload (N=1): the Wan-2.1-1.3B-shaped attention projection as an NVFP4
W4A4 linear layer, A bf16 [32760, 1536] (N(0,1) with 0.1% x50 outliers),
W [1536, 1536] ~N(0, 1/sqrt(1536)), bias [1536] ~N(0, 0.01), static activation
scale 1.0; the weight is quantized once before timing (load time).  One step =
quantize A (NVFP4 kernel) + block-scaled GEMM with alpha and bias fused (tcgen05
kernel), inputs resident in HBM; the K timed steps are replayed as one CUDA graph
with timing events recorded as graph nodes around each step (the per-kernel split
comes from a second graph with an event between the two kernels).
`value` = 2*M*N*K per step / step time (TFLOP/s) summed over ranks; L2 is
flushed (256 MiB write) before every timed step, outside the timed events.

Other --config values (wan14_in, wan14_out, mxfp8, skinny_m<M>, tiny) time the
corresponding workload the same way; --config loadtime times the load-time
conversion of the 240 weights of a 40-block DiT stack (GB/s).

--impl reference times the CPU oracle (oracle/, plain C + numpy float64) on a
bounded row sample of the same workload, on the host cores.

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
    "nvfp4_quantize": ("quantize.cu", "bsp_device.cuh", "bsp_internal.h"),
    "nvfp4_rmsnorm_quantize": ("quantize.cu", "bsp_device.cuh", "bsp_internal.h"),
    "mxfp8_quantize": ("quantize.cu", "bsp_device.cuh", "bsp_internal.h"),
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
def make_workload(name: str):
    from block_scaled_precision_05_b200 import workloads as wl
    if name == "wan13":
        return wl.wan13(), "nvfp4"
    if name == "tiny":
        return wl.tiny(), "nvfp4"
    if name in ("wan14_in", "wan14_out"):
        return getattr(wl, name)(), "nvfp4"
    if name == "mxfp8":
        return wl.mxfp8(), "mxfp8"
    if name.startswith("skinny_m"):
        return wl.skinny(int(name[len("skinny_m"):])), "nvfp4"
    raise SystemExit(f"unknown --config {name}")


NORM_EPS = 1e-6


def norm_gamma(lin):
    """Seeded RMSNorm weight for --norm rmsnorm: 1 + 0.2 N(0, 1), bf16 bits."""
    from block_scaled_precision_05_b200 import workloads as wl
    rng = np.random.default_rng(77)
    return wl.f32_to_bf16_bits((1.0 + 0.2 * rng.standard_normal(lin.K)).astype(np.float32))


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


def describe(lin, kind):
    d = {"workload": f"{lin.name}: {kind.upper()} linear A[{lin.M},{lin.K}] x W[{lin.N},{lin.K}]^T"
                     + (" + bias" if lin.bias is not None else "")
                     + (" (per-token activation scales)" if lin.per_token else ""),
         "M": lin.M, "N": lin.N, "K": lin.K,
         "l2": "flushed before every timed step (256 MiB write, outside the timed events)",
         "timing": "K steps in one CUDA graph, CUDA events as graph nodes around each step's two kernels; "
                   "per-kernel split from a second graph with an event also between them"}
    return d


def quant_bytes(M, K, kind, sf_layout="128x4"):
    """Algorithmic HBM bytes of one activation quantize launch."""
    if kind == "nvfp4":
        row_tile = 8 if sf_layout == "8x4" else 128
        return M * K * 2 + M * K // 2 + (-(-M // row_tile) * row_tile) * (-(-(K // 16) // 4) * 4)
    return M * K * 2 + M * K + (-(-M // 128) * 128) * (-(-(K // 32) // 4) * 4)


# --------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from block_scaled_precision_05_b200 import api

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    lin, kind = make_workload(args.config)
    lin = apply_input_format(lin, kind, args.input)
    a_dtype = torch.float16 if lin.fmt == "f16" else torch.bfloat16

    def up(a, dtype=torch.bfloat16):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(dtype).to(dev)

    A = up(lin.A, a_dtype)
    if args.norm == "rmsnorm":
        if kind != "nvfp4" or lin.fmt != "bf16":
            raise SystemExit("--norm rmsnorm applies to the bf16 NVFP4 workloads")
        gamma = up(norm_gamma(lin))
    W = up(lin.W)
    bias = None if lin.bias is None else up(lin.bias)
    if kind == "nvfp4":
        layer = api.NVFP4Linear(W, bias, per_token=lin.per_token, four_over_six=args.four_over_six)
    else:
        layer = api.MXFP8Linear(W, bias)
    del W
    M, N, K = lin.M, lin.N, lin.K
    flops = 2.0 * M * N * K
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    # preallocated outputs: the timed step launches exactly our two kernels
    if kind == "nvfp4":
        if args.sf_layout == "8x4" and (M > 64 or args.norm == "rmsnorm"):
            raise SystemExit("--sf-layout 8x4 applies to NVFP4 workloads with M <= 64 and no fused norm")
        xq = api.NVFP4Tensor(torch.empty((M, K // 2), dtype=torch.uint8, device=dev),
                             torch.empty(api.nvfp4_sf_bytes(M, K, args.sf_layout), dtype=torch.uint8, device=dev), K,
                             sf_layout=args.sf_layout)
        if lin.per_token:
            xq.row_gs = torch.empty(M, dtype=torch.float32, device=dev)
            xq.row_inv_gs = torch.empty(M, dtype=torch.float32, device=dev)
    else:
        xq = api.MXFP8Tensor(torch.empty((M, K), dtype=torch.uint8, device=dev),
                             torch.empty(api.mxfp8_sf_bytes(M, K), dtype=torch.uint8, device=dev), K)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=dev)

    def quantize():
        if args.norm == "rmsnorm":
            api.nvfp4_rmsnorm_quantize(A, gamma, NORM_EPS, None if lin.per_token else layer.gs_x,
                                       per_row=lin.per_token, out=xq)
        elif kind == "nvfp4":
            api.nvfp4_quantize(A, None if lin.per_token else layer.gs_x, per_row=lin.per_token, out=xq,
                               sf_layout=args.sf_layout)
        else:
            api.mxfp8_quantize(A, out=xq)

    def gemm():
        if kind == "nvfp4":
            api.nvfp4_gemm(xq, layer.weight, layer.alpha, xq.row_inv_gs if lin.per_token else None, layer.bias,
                           out=D)
        else:
            api.mxfp8_gemm(xq, layer.weight, None, layer.bias, out=D)

    for _ in range(args.warmup):
        flush.zero_()
        quantize()
        gemm()
    torch.cuda.synchronize()
    if api.device_status() != 0:
        raise RuntimeError("device error word set during warm-up")

    # The timed region is one CUDA graph holding all K steps back to back: per
    # step an L2 flush, then a timing event, the quantize and GEMM launches and a
    # second timing event (events are graph nodes; no Python/ctypes launch
    # latency inside the measured intervals).  The library is capturable (no
    # allocation, no host synchronisation).  A second graph of the same steps
    # with an event also between the two kernels gives the per-kernel split for
    # the roofline; every event interval on this device carries a launch floor
    # of about 6 us (an empty kernel between two event nodes reads 6.1 us).
    def step(evs, split):  # records on the current (capturing) stream
        flush.zero_()
        evs[0].record()
        quantize()
        if split:
            evs[1].record()
        gemm()
        evs[2].record()

    def graph_of(steps, split):
        evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(steps)]
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
    step_ms = [ev[s][0].elapsed_time(ev[s][2]) for s in range(args.steps)]
    t_q = [ev_split[s][0].elapsed_time(ev_split[s][1]) for s in range(args.steps)]
    t_g = [ev_split[s][1].elapsed_time(ev_split[s][2]) for s in range(args.steps)]
    total_ms = float(sum(step_ms))
    total_ms = max_over_ranks(total_ms, world, dev)
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
    def launches_for(step_ms):
        return int(min(24, max(4, 2.0 / max(step_ms, 1e-3))))

    q_step_ms, g_step_ms = statistics.mean(t_q), statistics.mean(t_g)
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size

    def rotations(streamed_bytes):
        return int(min(8, max(2, -(-3 * l2_bytes // max(1, streamed_bytes)))))

    def back_to_back(launch, n_rot, R):
        for r in range(n_rot):
            launch(r)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for r in range(R):
                launch(r % n_rot)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g.replay()
        torch.cuda.synchronize()
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) / R

    # the GEMM streams A (large M) or the weight (skinny M) from DRAM
    w_bytes = layer.weight.codes.numel() + layer.weight.sf.numel() if kind == "nvfp4" else \
        layer.weight.q.numel() + layer.weight.sf.numel()
    a_bytes = xq.codes.numel() + xq.sf.numel() if kind == "nvfp4" else xq.q.numel() + xq.sf.numel()
    rotate_weight = w_bytes > a_bytes
    nq = rotations(A.numel() * A.element_size())  # bf16 inputs of the quantizer
    nx = max(nq, 1 if rotate_weight else rotations(a_bytes))  # quantized activations
    A_rot = [A] + [A.clone() for _ in range(nq - 1)]
    if kind == "nvfp4":
        xq_rot = [xq] + [api.NVFP4Tensor(torch.empty_like(xq.codes), torch.empty_like(xq.sf), K,
                                          sf_layout=xq.sf_layout) for _ in range(nx - 1)]
        for t in xq_rot[1:]:
            if lin.per_token:
                t.row_gs, t.row_inv_gs = torch.empty_like(xq.row_gs), torch.empty_like(xq.row_inv_gs)
    else:
        xq_rot = [xq] + [api.MXFP8Tensor(torch.empty_like(xq.q), torch.empty_like(xq.sf), K) for _ in range(nx - 1)]

    def quant_launch(r):
        x, out = A_rot[r % nq], xq_rot[r]
        if args.norm == "rmsnorm":
            api.nvfp4_rmsnorm_quantize(x, gamma, NORM_EPS, None if lin.per_token else layer.gs_x,
                                       per_row=lin.per_token, out=out)
        elif kind == "nvfp4":
            api.nvfp4_quantize(x, None if lin.per_token else layer.gs_x, per_row=lin.per_token, out=out,
                               sf_layout=args.sf_layout)
        else:
            api.mxfp8_quantize(x, out=out)

    R_q, R_g = launches_for(q_step_ms), launches_for(g_step_ms)
    q_b2b_ms = back_to_back(quant_launch, nx, max(R_q, nx))  # also fills every quantized buffer
    ng = rotations(max(w_bytes, a_bytes))
    if rotate_weight:
        w = layer.weight
        if kind == "nvfp4":
            w_rot = [w] + [api.NVFP4Tensor(w.codes.clone(), w.sf.clone(), K) for _ in range(ng - 1)]
        else:
            w_rot = [w] + [api.MXFP8Tensor(w.q.clone(), w.sf.clone(), K) for _ in range(ng - 1)]
    D_rot = [D] + [torch.empty_like(D) for _ in range(min(ng, 2) - 1)]

    def gemm_launch(r):
        a = xq if rotate_weight else xq_rot[r]
        b = w_rot[r] if rotate_weight else layer.weight
        out = D_rot[r % len(D_rot)]
        if kind == "nvfp4":
            api.nvfp4_gemm(a, b, layer.alpha, a.row_inv_gs if lin.per_token else None, layer.bias, out=out)
        else:
            api.mxfp8_gemm(a, b, None, layer.bias, out=out)

    g_b2b_ms = back_to_back(gemm_launch, ng if rotate_weight else nx, R_g)
    del A_rot, xq_rot, D_rot
    if rotate_weight:
        del w_rot
    q_b2b_ms = max_over_ranks(q_b2b_ms, world, dev)
    g_b2b_ms = max_over_ranks(g_b2b_ms, world, dev)

    # ---- end to end through the public API: every step copies its input from
    # pinned host memory and its result back to pinned host memory.  With large
    # copies the steps are pipelined as a serving loop would run them: the
    # copy-in of step i+1 and the copy-out of step i-1 run on their own streams
    # while step i computes (two device input buffers, two host output
    # buffers).  With small copies (skinny M) the extra stream bookkeeping costs
    # more host time than it hides, and the steps run on one stream.
    A_host = torch.from_numpy(np.ascontiguousarray(lin.A).view(np.int16)).view(a_dtype).pin_memory()
    D_host = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    A_dev = [torch.empty_like(A) for _ in range(2)]
    e2e_steps = max(2, min(args.steps, 20))
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]

    pipelined = A.numel() * 2 + M * N * 2 > (16 << 20)

    def e2e_step(i):
        b = i % 2
        if not pipelined:
            A_dev[0].copy_(A_host, non_blocking=True)
            if args.norm == "rmsnorm":
                y = layer(A_dev[0], pre_quantized=layer.rmsnorm_quantize_input(A_dev[0], gamma, NORM_EPS))
            else:
                y = layer(A_dev[0], sf_layout=args.sf_layout) if kind == "nvfp4" else layer(A_dev[0])
            D_host[0].copy_(y, non_blocking=True)
            return
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_comp[b])  # step i-2 has finished reading A_dev[b]
            A_dev[b].copy_(A_host, non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        if args.norm == "rmsnorm":
            y = layer(A_dev[b], pre_quantized=layer.rmsnorm_quantize_input(A_dev[b], gamma, NORM_EPS))
        else:
            y = layer(A_dev[b], sf_layout=args.sf_layout) if kind == "nvfp4" else layer(A_dev[b])
        ev_comp[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            D_host[b].copy_(y, non_blocking=True)  # in order after step i-2's copy of D_host[b]
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
    q_ms, g_ms = q_b2b_ms, g_b2b_ms
    qb = quant_bytes(M, K, kind, args.sf_layout)
    q_gbs = qb / (q_ms * 1e-3) / 1e9
    g_tflops = flops / (g_ms * 1e-3) / 1e12
    ratio = FP4_PER_BF16 if kind == "nvfp4" else FP8_PER_BF16
    tensor_peak = peaks["bf16_tflops"] * ratio
    hbm_peak = peaks["hbm_gbs"]
    wname = args.config + ("_rmsnorm" if args.norm == "rmsnorm" else "")
    qname = "nvfp4_rmsnorm_quantize" if args.norm == "rmsnorm" else f"{kind}_quantize"
    if M <= 128:
        # skinny M: the GEMM streams the weight once; bound by HBM
        gb = (M * K + N * K) * (0.5 if kind == "nvfp4" else 1.0) + (M + N) * (K // 16 if kind == "nvfp4" else K // 32) \
            + 2 * M * N
        g_gbs = gb / (g_ms * 1e-3) / 1e9
        roof = {"kernel": f"{kind}_gemm", "bound": "hbm", "achieved": round(g_gbs, 1), "peak": hbm_peak,
                "unit": "GB/s", "frac": round(g_gbs / hbm_peak, 4), "traffic": traffic_for(f"{kind}_gemm", wname),
                "peak_source": f"{peak_src}: hbm_gbs",
                "algorithmic": f"{int(gb)} bytes per launch (operand codes + scales + output)"}
    elif g_ms >= q_ms:
        roof = {"kernel": f"{kind}_gemm", "bound": "tensor", "achieved": round(g_tflops, 1),
                "peak": round(tensor_peak, 1), "unit": "TFLOP/s", "frac": round(g_tflops / tensor_peak, 4),
                "traffic": traffic_for(f"{kind}_gemm", wname),
                "peak_source": f"{peak_src}: bf16_tflops (burst) x {ratio:g} nominal {kind} ratio",
                "algorithmic": f"2*M*N*K = {flops:.4g} flop per launch"}
    else:
        roof = {"kernel": qname, "bound": "hbm", "achieved": round(q_gbs, 1), "peak": hbm_peak,
                "unit": "GB/s", "frac": round(q_gbs / hbm_peak, 4), "traffic": traffic_for(qname, wname),
                "peak_source": f"{peak_src}: hbm_gbs", "algorithmic": f"{qb} bytes per launch"}

    cfg = describe(lin, kind)
    cfg["parallelism"] = f"replicas x{world}"
    cfg["activation_dtype"] = "fp16" if lin.fmt == "f16" else "bf16"
    if kind == "nvfp4":
        cfg["activation_sf_layout"] = args.sf_layout
    if args.norm == "rmsnorm":
        cfg["producer"] = f"RMSNorm (gamma 1+0.2N(0,1), eps {NORM_EPS:g}) fused into the quantizer"
    if kind == "nvfp4":
        cfg["weight_global_scale"] = "256*6/amax (4over6)" if args.four_over_six else "448*6/amax"
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4" if kind == "nvfp4" else "mxfp8", "data": "synthetic (seeded numpy)",
        "config": cfg, "roofline": roof,
        "kernels": {
            qname: {"ms": round(q_ms, 5), "GB/s": round(q_gbs, 1), "frac_hbm": round(q_gbs / hbm_peak, 4)},
            f"{kind}_gemm": {"ms": round(g_ms, 5), "TFLOP/s": round(g_tflops, 1),
                             "frac_tensor_peak": round(g_tflops / tensor_peak, 4)},
            "timing": f"{R_q} / {R_g} launches back to back in one CUDA graph between two events (about 2 ms), "
                      "operands rotated through buffers totalling > 3x L2 so each launch streams from DRAM",
            "per_step_event_split_ms": {qname: round(q_step_ms, 5), f"{kind}_gemm": round(g_step_ms, 5),
                                        "note": "events around each kernel inside the timed steps; each "
                                                "interval carries a ~6 us event/launch floor"},
        },
        "e2e": {"value": round(whole_job_rate(flops, world, 1, e2e_ms) / 1e12, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(A_host.numel() * 2), "d2h_bytes_per_step": int(D_host[0].numel() * 2),
                "ms_per_step": round(e2e_ms, 4), "runs_ms_per_step": [round(v, 4) for v in e2e_runs],
                "steps_per_run": e2e_steps,
                "pipelining": ("each step's copy-in, compute and copy-out on three streams; consecutive steps "
                               "overlap") if pipelined else "none (one stream; small copies)"},
        "gpu_launches": 2 * args.steps,
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = oracle_baseline(lin, kind, budget_s=args.cpu_budget, four_over_six=args.four_over_six,
                                              norm=args.norm)
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
    """The oracle's linear layer on `rows` of A: quantize, decode, float64 GEMM, epilogue."""
    import oracle
    K = lin.K
    A = lin.A[rows]
    if kind == "nvfp4":
        gs_w, codes_b, sf_b, decB = wq
        fmt = getattr(lin, "fmt", "bf16")
        if norm == "rmsnorm":
            A = oracle.rmsnorm_bf16(A, norm_gamma(lin), oracle.rmsnorm_rstd(A, NORM_EPS))
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


def oracle_baseline(lin, kind, budget_s=10.0, four_over_six=False, norm=None):
    """Times the oracle on a bounded row sample, scaled to TFLOP/s."""
    wq = oracle_weights(lin, kind, four_over_six)
    rng = np.random.default_rng(123)
    rows = np.sort(rng.choice(lin.M, size=min(lin.M, 128), replace=False))
    t0 = time.perf_counter()
    oracle_step(lin, kind, rows, wq, norm)
    dt = time.perf_counter() - t0
    n = int(min(lin.M, max(128, 128 * budget_s / max(dt, 1e-3))))
    rows = np.sort(rng.choice(lin.M, size=n, replace=False))
    t0 = time.perf_counter()
    oracle_step(lin, kind, rows, wq, norm)
    dt = time.perf_counter() - t0
    flops = 2.0 * n * lin.N * lin.K
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": max(os.cpu_count() or 1, blas_threads()),
            "kind": "oracle", "seconds": round(dt, 2),
            "sample": f"{n} random rows of A (of {lin.M}): quantize + decode + float64 GEMM + epilogue + bf16 "
                      f"rounding; weight quantized beforehand (load time)"}


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
    if args.config == "loadtime":
        return run_reference_loadtime(args)
    lin, kind = make_workload(args.config)
    lin = apply_input_format(lin, kind, args.input)
    wq = oracle_weights(lin, kind, args.four_over_six)
    rng = np.random.default_rng(7)
    n = min(lin.M, args.ref_rows)
    for _ in range(args.warmup):
        oracle_step(lin, kind, np.sort(rng.choice(lin.M, size=n, replace=False)), wq, args.norm)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(lin, kind, np.sort(rng.choice(lin.M, size=n, replace=False)), wq, args.norm)
    dt = time.perf_counter() - t0
    flops = 2.0 * n * lin.N * lin.K * args.steps
    value = flops / dt / 1e12
    cores = max(os.cpu_count() or 1, blas_threads())
    sample = (f"{n} random rows of A per step (of {lin.M}): quantize + decode + float64 GEMM + epilogue + bf16 "
              f"rounding; weight quantized beforehand (load time)")
    cfg = describe(lin, kind)
    cfg["parallelism"] = "host cores"
    cfg["activation_dtype"] = "fp16" if lin.fmt == "f16" else "bf16"
    if kind == "nvfp4":
        cfg["activation_sf_layout"] = args.sf_layout
    if args.norm == "rmsnorm":
        cfg["producer"] = f"RMSNorm (gamma 1+0.2N(0,1), eps {NORM_EPS:g}) fused into the quantizer"
    if kind == "nvfp4":
        cfg["weight_global_scale"] = "256*6/amax (4over6)" if args.four_over_six else "448*6/amax"
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64 (oracle)", "data": "synthetic (seeded numpy)", "config": cfg,
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# --------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="wan13")
    ap.add_argument("--sf-layout", choices=["128x4", "8x4"], default="128x4",
                    help="activation scale layout of the NVFP4 workloads (8x4: M <= 64)")
    ap.add_argument("--norm", choices=["none", "rmsnorm"], default="none",
                    help="NVFP4 workloads: fuse an RMSNorm of the activation into the quantizer")
    ap.add_argument("--input", choices=["bf16", "f16"], default="bf16",
                    help="activation dtype of the NVFP4 workloads (f16: the bf16 values rounded to fp16)")
    ap.add_argument("--four-over-six", action="store_true",
                    help="NVFP4 weight global scale 256*6/amax (the 4over6 setting) instead of 448*6/amax")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-rows", type=int, default=256, help="rows per oracle step for --impl reference")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--blocks", type=int, default=40, help="DiT blocks for --config loadtime")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

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
