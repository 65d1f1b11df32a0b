"""PyTorch-facing API over the C ABI (include/bsp.h).

PyTorch provides device memory and the current stream; every step of the
quantize / GEMM path runs in libbsp's CUDA kernels.  Functions here only check
arguments, allocate outputs and pass pointers.

Sources (page title, then symbol):
  hao-ai-lab-FastVideo nvfp4_qat_config.py -- NVFP4QATQuantizeMethod.apply
      (flatten to [-1, K], quantize with the static activation scale 1.0,
      mm_fp4 with alpha = 1/(gs_x*gs_w), add bias, restore leading dims);
      convert_model_to_fp4 (weight amax -> gs_w = 448*6/amax -> quantize).
  hao-ai-lab-FastVideo nvfp4_config.py -- _coerce_fp4_input_dtype (fp32 input
      is cast to bf16, non-float input is a TypeError), the register_fake
      shapes of nvfp4_quantize ([M, K/2] codes) and mm_fp4 ([*a.shape[:-1], N]).
  sglang nvfp4_online.py -- per-token activation scales; the all-zero weight
      guard (scale 1 when amax is 0); K % 16 == 0 and 2-D weights required.
  vllm-omni mxfp8_config.py -- MXFPLinearMethodBase.apply (reshape, quantize
      the activation with one e8m0 scale per 32, GEMM with bias, reshape).
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _native as nat


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _require_cuda(*ts: torch.Tensor | None) -> None:
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libbsp runs on CUDA tensors only (no CPU path)")


def coerce_input(x: torch.Tensor) -> torch.Tensor:
    """Input dtype rule of the NVFP4 path (nvfp4_config.py,
    _coerce_fp4_input_dtype): bf16 and fp16 pass as they are, other floats are
    cast to bf16, anything else is an error."""
    if not x.is_floating_point():
        raise TypeError(f"block-scaled linear expects floating-point inputs, got {x.dtype}")
    return x if x.dtype in (torch.bfloat16, torch.float16) else x.to(torch.bfloat16)


def coerce_bf16(x: torch.Tensor) -> torch.Tensor:
    """bf16 for the paths whose kernels read bf16 only (MXFP8, the bias)."""
    if not x.is_floating_point():
        raise TypeError(f"block-scaled linear expects floating-point inputs, got {x.dtype}")
    return x if x.dtype == torch.bfloat16 else x.to(torch.bfloat16)


_HALF_TYPES = (torch.bfloat16, torch.float16)


def nvfp4_sf_bytes(rows: int, K: int, sf_layout: str = "128x4") -> int:
    return int(nat.lib().bsp_nvfp4_sf_bytes_layout(rows, K, SF_LAYOUTS[sf_layout]))


def mxfp8_sf_bytes(rows: int, K: int) -> int:
    return int(nat.lib().bsp_mxfp8_sf_bytes(rows, K))


# --------------------------------------------------------------------------- scales
# e4m3_max * 6: the numerator of the NVFP4 global scale.  448 is the largest
# e4m3 value; the 4over6 setting of nvfp4_online.py _quantize_weight_nvfp4 uses
# 256 so that every group scale stays <= 256.
FP8_FP4_MAX = 448.0 * 6.0
FP8_FP4_MAX_4OVER6 = 256.0 * 6.0


def amax(x: torch.Tensor) -> torch.Tensor:
    """fp32 [1] device tensor: max |x| over a bf16 or fp16 tensor (NaN as 0, inf
    as the format's largest finite value)."""
    _require_cuda(x)
    if x.dtype not in _HALF_TYPES or not x.is_contiguous():
        raise ValueError("amax expects a contiguous bf16 or fp16 tensor")
    out = torch.empty(1, dtype=torch.float32, device=x.device)
    fn = "bsp_amax_bf16" if x.dtype == torch.bfloat16 else "bsp_amax_f16"
    nat.check(getattr(nat.lib(), fn)(_ptr(x), x.numel(), _ptr(out), _stream()), fn)
    return out


def amax_into(x: torch.Tensor, out: torch.Tensor) -> torch.Tensor:
    """Folds max |x| into `out` (an fp32 [1] amax from `amax`) on the device."""
    _require_cuda(x, out)
    if x.dtype not in _HALF_TYPES or not x.is_contiguous():
        raise ValueError("amax_into expects a contiguous bf16 or fp16 tensor")
    if out.dtype != torch.float32 or out.numel() != 1:
        raise ValueError("amax_into expects an fp32 [1] accumulator")
    fn = "bsp_amax_bf16_into" if x.dtype == torch.bfloat16 else "bsp_amax_f16_into"
    nat.check(getattr(nat.lib(), fn)(_ptr(x), x.numel(), _ptr(out), _stream()), fn)
    return out


def nvfp4_global_scale(amax_t: torch.Tensor, fp8_fp4_max: float = FP8_FP4_MAX) -> tuple[torch.Tensor, torch.Tensor]:
    """(gs, 1/gs) fp32 [1] device tensors with gs = fp8_fp4_max/amax (1 for amax 0)."""
    _require_cuda(amax_t)
    gs = torch.empty(1, dtype=torch.float32, device=amax_t.device)
    inv = torch.empty_like(gs)
    nat.check(nat.lib().bsp_nvfp4_global_scale_max(_ptr(amax_t), float(fp8_fp4_max), _ptr(gs), _ptr(inv), _stream()),
              "bsp_nvfp4_global_scale_max")
    return gs, inv


def nvfp4_quantize_shared(weights, fp8_fp4_max: float = FP8_FP4_MAX):
    """Quantizes several bf16 weights with one global scale from their joint
    amax (the gated w1/w3 pair of nvfp4_online.py, quantized together so both
    halves share one per-tensor scale).  Returns ([NVFP4Tensor], gs, 1/gs)."""
    ws = [coerce_input(w).contiguous() for w in weights]
    if not ws:
        raise ValueError("nvfp4_quantize_shared needs at least one weight")
    a = amax(ws[0])
    for w in ws[1:]:
        amax_into(w, a)
    gs, inv = nvfp4_global_scale(a, fp8_fp4_max)
    return [nvfp4_quantize(w, gs) for w in ws], gs, inv


def nvfp4_alpha(gs_x: torch.Tensor, gs_w: torch.Tensor) -> torch.Tensor:
    """alpha = 1/(gs_x * gs_w), fp32 [1] device tensor."""
    _require_cuda(gs_x, gs_w)
    out = torch.empty(1, dtype=torch.float32, device=gs_x.device)
    nat.check(nat.lib().bsp_nvfp4_alpha(_ptr(gs_x), _ptr(gs_w), _ptr(out), _stream()), "bsp_nvfp4_alpha")
    return out


# --------------------------------------------------------------------------- quantize
SF_LAYOUTS = {"128x4": nat.BSP_SF_LAYOUT_128X4, "8x4": nat.BSP_SF_LAYOUT_8X4}


@dataclass
class NVFP4Tensor:
    """Packed NVFP4 rows: codes uint8 [M, K/2], scales uint8 in the 128x4 (or,
    for small M, 8x4) tile layout."""
    codes: torch.Tensor
    sf: torch.Tensor
    K: int
    row_gs: torch.Tensor | None = None      # per-row encode scales (PER_ROW)
    row_inv_gs: torch.Tensor | None = None  # per-row decode factors 1/gs (PER_ROW)
    sf_layout: str = "128x4"

    @property
    def rows(self) -> int:
        return self.codes.shape[0]


@dataclass
class MXFP8Tensor:
    """MXFP8 rows: e4m3 bytes [M, K], e8m0 scales (128x4 layout)."""
    q: torch.Tensor
    sf: torch.Tensor
    K: int

    @property
    def rows(self) -> int:
        return self.q.shape[0]


def _as_2d(x: torch.Tensor) -> torch.Tensor:
    x2 = x.reshape(-1, x.shape[-1])
    if x2.stride(-1) != 1:
        x2 = x2.contiguous()
    return x2


def nvfp4_quantize(x: torch.Tensor, global_sf: torch.Tensor | None = None, per_row: bool = False,
                   out: NVFP4Tensor | None = None, sf_layout: str = "128x4") -> NVFP4Tensor:
    """Quantize bf16 or fp16 [..., K] to NVFP4 along K (leading dims flattened).
    sf_layout "8x4" stores the scales in 8-row tiles (small M; nvfp4_gemm then
    takes them for M <= 64)."""
    _require_cuda(x, global_sf)
    if x.dtype not in _HALF_TYPES:
        raise TypeError("nvfp4_quantize expects bf16 or fp16 input (use coerce_input first)")
    x2 = _as_2d(x)
    M, K = x2.shape
    dev = x2.device
    if sf_layout not in SF_LAYOUTS:
        raise ValueError(f"sf_layout must be one of {sorted(SF_LAYOUTS)}")
    if out is None:
        out = NVFP4Tensor(torch.empty((M, K // 2), dtype=torch.uint8, device=dev),
                          torch.empty(nvfp4_sf_bytes(M, K, sf_layout), dtype=torch.uint8, device=dev), K,
                          sf_layout=sf_layout)
        if per_row:
            out.row_gs = torch.empty(M, dtype=torch.float32, device=dev)
            out.row_inv_gs = torch.empty(M, dtype=torch.float32, device=dev)
    elif out.sf_layout != sf_layout:
        raise ValueError("out was allocated for another scale layout")
    if not per_row and global_sf is None:
        raise ValueError("per-tensor quantization needs global_sf (fp32 device tensor)")
    st = nat.lib().nvfp4_quantize_ex(
        _ptr(x2), nat.BSP_IN_BF16 if x2.dtype == torch.bfloat16 else nat.BSP_IN_F16, M, K, x2.stride(0),
        None if per_row else _ptr(global_sf), nat.BSP_SF_PER_ROW if per_row else nat.BSP_SF_PER_TENSOR,
        SF_LAYOUTS[sf_layout], _ptr(out.row_gs) if per_row else None, _ptr(out.row_inv_gs) if per_row else None,
        _ptr(out.codes), _ptr(out.sf), _stream())
    nat.check(st, "nvfp4_quantize_ex")
    return out


# one zero-initialised workspace per (device, input format), created on first use
_WEIGHT_WS: dict[tuple[int, int], torch.Tensor] = {}


def _weight_workspace(device: torch.device, w_dtype: int) -> torch.Tensor:
    idx = device.index if device.index is not None else torch.cuda.current_device()
    ws = _WEIGHT_WS.get((idx, w_dtype))
    if ws is None:
        if torch.cuda.is_current_stream_capturing():
            raise RuntimeError("nvfp4_quantize_weight: the first call on a device sets up its workspace and must "
                               "not be inside a CUDA graph capture")
        n = ctypes.c_int64(0)
        with torch.cuda.device(idx):
            nat.check(nat.lib().bsp_nvfp4_quantize_weight_workspace_bytes(w_dtype, ctypes.addressof(n)),
                      "bsp_nvfp4_quantize_weight_workspace_bytes")
        ws = torch.zeros(n.value, dtype=torch.uint8, device=torch.device("cuda", idx))
        _WEIGHT_WS[(idx, w_dtype)] = ws
    return ws


def nvfp4_quantize_weight(w: torch.Tensor, fp8_fp4_max: float = FP8_FP4_MAX, out: NVFP4Tensor | None = None):
    """Load-time weight conversion in one kernel: amax, gs = fp8_fp4_max/amax and
    the per-tensor NVFP4 quantization with gs, bit-identical to amax ->
    nvfp4_global_scale -> nvfp4_quantize.  bf16 or fp16 [N, K], K % 64 == 0.
    Returns (NVFP4Tensor, gs, 1/gs, amax), the scalars fp32 [1] device tensors.
    The kernel's workspace is kept per device; calls on one device must not
    overlap in time (one stream, or ordered streams)."""
    _require_cuda(w)
    w = coerce_input(w)
    if w.dim() != 2 or w.shape[1] % 64 != 0 or w.shape[0] == 0:
        raise ValueError(f"nvfp4_quantize_weight expects [N, K] with N > 0 and K % 64 == 0, got {tuple(w.shape)}")
    if w.stride(1) != 1:
        w = w.contiguous()
    N, K = w.shape
    dev = w.device
    if out is None:
        out = NVFP4Tensor(torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                          torch.empty(nvfp4_sf_bytes(N, K), dtype=torch.uint8, device=dev), K)
    gs, inv, am = (torch.empty(1, dtype=torch.float32, device=dev) for _ in range(3))
    w_dtype = nat.BSP_IN_F16 if w.dtype == torch.float16 else nat.BSP_IN_BF16
    ws = _weight_workspace(dev, w_dtype)
    nat.check(nat.lib().nvfp4_quantize_weight(_ptr(w), w_dtype, N, K, w.stride(0), float(fp8_fp4_max), _ptr(am),
                                              _ptr(gs), _ptr(inv), _ptr(out.codes), _ptr(out.sf), _ptr(ws),
                                              ws.numel(), _stream()), "nvfp4_quantize_weight")
    return out, gs, inv, am


def nvfp4_quantize_weights(weights, fp8_fp4_max: float = FP8_FP4_MAX):
    """nvfp4_quantize_weight for a list of [N, K] weights of one dtype (K % 64
    == 0), up to BSP_WEIGHT_BATCH_MAX per launch: the load-time conversion of a
    model's linears in one cooperative launch per chunk.  Returns one
    (NVFP4Tensor, gs, 1/gs, amax) per weight, bit-identical to
    nvfp4_quantize_weight on it."""
    ws_in = []
    for w in weights:
        _require_cuda(w)
        w = coerce_input(w)
        if w.dim() != 2 or w.shape[1] % 64 != 0 or w.shape[0] == 0:
            raise ValueError(f"nvfp4_quantize_weights expects [N, K] weights with N > 0 and K % 64 == 0, "
                             f"got {tuple(w.shape)}")
        ws_in.append(w if w.stride(1) == 1 else w.contiguous())
    if not ws_in:
        return []
    dtypes = {w.dtype for w in ws_in}
    devices = {w.device for w in ws_in}
    if len(dtypes) != 1 or len(devices) != 1:
        raise ValueError("nvfp4_quantize_weights expects weights of one dtype on one device")
    dev = ws_in[0].device
    w_dtype = nat.BSP_IN_F16 if ws_in[0].dtype == torch.float16 else nat.BSP_IN_BF16
    work = _weight_workspace(dev, w_dtype)
    results = []
    for c0 in range(0, len(ws_in), nat.BSP_WEIGHT_BATCH_MAX):
        chunk = ws_in[c0:c0 + nat.BSP_WEIGHT_BATCH_MAX]
        descs = (nat.BspWeightDesc * len(chunk))()
        for d, w in zip(descs, chunk):
            N, K = w.shape
            q = NVFP4Tensor(torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                            torch.empty(nvfp4_sf_bytes(N, K), dtype=torch.uint8, device=dev), K)
            gs, inv, am = (torch.empty(1, dtype=torch.float32, device=dev) for _ in range(3))
            d.w, d.N, d.K, d.ld_w = w.data_ptr(), N, K, w.stride(0)
            d.amax, d.gs, d.inv_gs, d.codes, d.sf = am.data_ptr(), gs.data_ptr(), inv.data_ptr(), \
                q.codes.data_ptr(), q.sf.data_ptr()
            results.append((q, gs, inv, am))
        nat.check(nat.lib().nvfp4_quantize_weights(ctypes.addressof(descs), len(chunk), w_dtype, float(fp8_fp4_max),
                                                   _ptr(work), work.numel(), _stream()), "nvfp4_quantize_weights")
    return results


def nvfp4_rmsnorm_quantize(x: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-6,
                           global_sf: torch.Tensor | None = None, per_row: bool = False,
                           out: NVFP4Tensor | None = None, rstd_out: torch.Tensor | None = None) -> NVFP4Tensor:
    """RMSNorm(x) * gamma, rounded to bf16 and quantized to NVFP4 in one kernel
    (the normalised activation is never written).  bf16 x [..., K], gamma [K]."""
    _require_cuda(x, gamma, global_sf, rstd_out)
    if x.dtype != torch.bfloat16 or gamma.dtype != torch.bfloat16:
        raise TypeError("nvfp4_rmsnorm_quantize expects bf16 x and gamma")
    x2 = _as_2d(x)
    M, K = x2.shape
    if gamma.numel() != K or not gamma.is_contiguous():
        raise ValueError(f"gamma must be a contiguous [{K}] tensor")
    if rstd_out is not None and (rstd_out.dtype != torch.float32 or rstd_out.numel() != M):
        raise ValueError(f"rstd_out must be an fp32 [{M}] tensor")
    dev = x2.device
    if out is None:
        out = NVFP4Tensor(torch.empty((M, K // 2), dtype=torch.uint8, device=dev),
                          torch.empty(nvfp4_sf_bytes(M, K), dtype=torch.uint8, device=dev), K)
        if per_row:
            out.row_gs = torch.empty(M, dtype=torch.float32, device=dev)
            out.row_inv_gs = torch.empty(M, dtype=torch.float32, device=dev)
    if not per_row and global_sf is None:
        raise ValueError("per-tensor quantization needs global_sf (fp32 device tensor)")
    st = nat.lib().nvfp4_rmsnorm_quantize(
        _ptr(x2), M, K, x2.stride(0), _ptr(gamma), float(eps), None if per_row else _ptr(global_sf),
        nat.BSP_SF_PER_ROW if per_row else nat.BSP_SF_PER_TENSOR,
        _ptr(out.row_gs) if per_row else None, _ptr(out.row_inv_gs) if per_row else None, _ptr(rstd_out),
        _ptr(out.codes), _ptr(out.sf), _stream())
    nat.check(st, "nvfp4_rmsnorm_quantize")
    return out


def nvfp4_layernorm_quantize(x: torch.Tensor, gamma: torch.Tensor | None = None, beta: torch.Tensor | None = None,
                             eps: float = 1e-6, global_sf: torch.Tensor | None = None, per_row: bool = False,
                             out: NVFP4Tensor | None = None, mean_out: torch.Tensor | None = None,
                             rstd_out: torch.Tensor | None = None) -> NVFP4Tensor:
    """LayerNorm(x) (* gamma + beta, each optional), rounded to bf16 and
    quantized to NVFP4 in one kernel (the normalised activation is never
    written).  bf16 x [..., K], gamma / beta [K] or None."""
    _require_cuda(x, gamma, beta, global_sf, mean_out, rstd_out)
    if x.dtype != torch.bfloat16 or any(t is not None and t.dtype != torch.bfloat16 for t in (gamma, beta)):
        raise TypeError("nvfp4_layernorm_quantize expects bf16 x, gamma and beta")
    x2 = _as_2d(x)
    M, K = x2.shape
    for name, t in (("gamma", gamma), ("beta", beta)):
        if t is not None and (t.numel() != K or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous [{K}] tensor")
    for name, t in (("mean_out", mean_out), ("rstd_out", rstd_out)):
        if t is not None and (t.dtype != torch.float32 or t.numel() != M):
            raise ValueError(f"{name} must be an fp32 [{M}] tensor")
    dev = x2.device
    if out is None:
        out = NVFP4Tensor(torch.empty((M, K // 2), dtype=torch.uint8, device=dev),
                          torch.empty(nvfp4_sf_bytes(M, K), dtype=torch.uint8, device=dev), K)
        if per_row:
            out.row_gs = torch.empty(M, dtype=torch.float32, device=dev)
            out.row_inv_gs = torch.empty(M, dtype=torch.float32, device=dev)
    if not per_row and global_sf is None:
        raise ValueError("per-tensor quantization needs global_sf (fp32 device tensor)")
    st = nat.lib().nvfp4_layernorm_quantize(
        _ptr(x2), M, K, x2.stride(0), _ptr(gamma), _ptr(beta), float(eps), None if per_row else _ptr(global_sf),
        nat.BSP_SF_PER_ROW if per_row else nat.BSP_SF_PER_TENSOR,
        _ptr(out.row_gs) if per_row else None, _ptr(out.row_inv_gs) if per_row else None, _ptr(mean_out),
        _ptr(rstd_out), _ptr(out.codes), _ptr(out.sf), _stream())
    nat.check(st, "nvfp4_layernorm_quantize")
    return out


def norm_stats(x: torch.Tensor, norm: str = "rms", exact_only: bool = False):
    """Diagnostic: the fused norms' row statistics alone (bsp_debug_norm_stats).
    Returns (ms,) for "rms" or (mean, var) for "layer", each fp32 [M], and the
    int32 [M] path flags (1 where the exact integer sums decided the row)."""
    _require_cuda(x)
    if x.dtype != torch.bfloat16:
        raise TypeError("norm_stats expects bf16 x")
    x2 = _as_2d(x)
    M, K = x2.shape
    dev = x2.device
    s0 = torch.empty(M, dtype=torch.float32, device=dev)
    s1 = torch.empty(M, dtype=torch.float32, device=dev) if norm == "layer" else None
    path = torch.empty(M, dtype=torch.int32, device=dev)
    kind = {"rms": nat.BSP_NORM_RMS, "layer": nat.BSP_NORM_LAYER}[norm]
    nat.check(nat.lib().bsp_debug_norm_stats(_ptr(x2), M, K, x2.stride(0), kind, int(exact_only), _ptr(s0), _ptr(s1),
                                             _ptr(path), _stream()), "bsp_debug_norm_stats")
    return ((s0,) if s1 is None else (s0, s1)), path


def mxfp8_quantize(x: torch.Tensor, out: MXFP8Tensor | None = None) -> MXFP8Tensor:
    """Quantize bf16 [..., K] to MXFP8 along K (leading dims flattened)."""
    _require_cuda(x)
    if x.dtype != torch.bfloat16:
        raise TypeError("mxfp8_quantize expects bf16 input (use coerce_input first)")
    x2 = _as_2d(x)
    M, K = x2.shape
    dev = x2.device
    if out is None:
        out = MXFP8Tensor(torch.empty((M, K), dtype=torch.uint8, device=dev),
                          torch.empty(mxfp8_sf_bytes(M, K), dtype=torch.uint8, device=dev), K)
    nat.check(nat.lib().mxfp8_quantize(_ptr(x2), M, K, x2.stride(0), _ptr(out.q), _ptr(out.sf), _stream()),
              "mxfp8_quantize")
    return out


# --------------------------------------------------------------------------- GEMM
def _out(M: int, N: int, dtype: torch.dtype, device, out: torch.Tensor | None) -> tuple[torch.Tensor, int]:
    if dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("output dtype must be bf16 or fp32")
    if out is None:
        out = torch.empty((M, N), dtype=dtype, device=device)
    if out.dtype != dtype or out.dim() != 2 or out.shape[0] != M or out.shape[1] != N or out.stride(1) != 1:
        raise ValueError("out must be a row-major [M, N] tensor of the output dtype")
    return out, (nat.BSP_OUT_F32 if dtype == torch.float32 else nat.BSP_OUT_BF16)


def _check_epilogue_args(alpha, row_scale, bias, N: int) -> None:
    for name, t in (("alpha", alpha), ("row_scale", row_scale)):
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous()):
            raise TypeError(f"{name} must be a contiguous fp32 device tensor")
    if bias is not None and (bias.dtype != torch.bfloat16 or not bias.is_contiguous() or bias.numel() != N):
        raise TypeError(f"bias must be a contiguous bf16 tensor of {N} elements")


def nvfp4_gemm(a: NVFP4Tensor, b: NVFP4Tensor, alpha: torch.Tensor | None = None,
               row_scale: torch.Tensor | None = None, bias: torch.Tensor | None = None,
               out_dtype: torch.dtype = torch.bfloat16, out: torch.Tensor | None = None) -> torch.Tensor:
    """D = alpha * row_scale[m] * (A (x) sfA)(B (x) sfB)^T + bias, fp32 accumulate."""
    if a.K != b.K:
        raise ValueError("A and B disagree on K")
    _require_cuda(a.codes, b.codes, alpha, row_scale, bias)
    M, N = a.rows, b.rows
    _check_epilogue_args(alpha, row_scale, bias, N)
    out, d_dtype = _out(M, N, out_dtype, a.codes.device, out)
    if b.sf_layout != "128x4":
        raise ValueError("the weight's scales must be in the 128x4 layout")
    st = nat.lib().nvfp4_gemm_ex(_ptr(a.codes), _ptr(a.sf), SF_LAYOUTS[a.sf_layout], _ptr(b.codes), _ptr(b.sf), M, N,
                                 a.K, _ptr(alpha), _ptr(row_scale), _ptr(bias), _ptr(out), d_dtype, out.stride(0),
                                 _stream())
    nat.check(st, "nvfp4_gemm_ex")
    return out


def mxfp8_gemm(a: MXFP8Tensor, b: MXFP8Tensor, alpha: torch.Tensor | None = None,
               bias: torch.Tensor | None = None, out_dtype: torch.dtype = torch.bfloat16,
               out: torch.Tensor | None = None) -> torch.Tensor:
    """D = alpha * (A (x) 2^sA)(B (x) 2^sB)^T + bias, fp32 accumulate."""
    if a.K != b.K:
        raise ValueError("A and B disagree on K")
    _require_cuda(a.q, b.q, alpha, bias)
    M, N = a.rows, b.rows
    _check_epilogue_args(alpha, None, bias, N)
    out, d_dtype = _out(M, N, out_dtype, a.q.device, out)
    st = nat.lib().mxfp8_gemm(_ptr(a.q), _ptr(a.sf), _ptr(b.q), _ptr(b.sf), M, N, a.K, _ptr(alpha), _ptr(bias),
                              _ptr(out), d_dtype, out.stride(0), _stream())
    nat.check(st, "mxfp8_gemm")
    return out


def device_status() -> int:
    """Synchronise the current stream and read/clear the device error word."""
    return int(nat.lib().bsp_device_status(_stream()))


# --------------------------------------------------------------------------- linear layers
class NVFP4Linear:
    """W4A4 NVFP4 linear layer: the weight is quantized once at construction
    (amax -> gs_w -> quantize, one kernel when K % 64 == 0; the bf16 weight is
    not kept), each call quantizes
    the activation and runs the block-scaled GEMM with alpha and bias fused.

    per_token=False: static activation scale gs_x = 1.0 (no reduction, no host
    sync, capturable in a CUDA graph).  per_token=True: per-row activation
    scales computed inside the quantize kernel and applied in the GEMM epilogue.
    four_over_six=True: weight global scale 256*6/amax instead of 448*6/amax
    (nvfp4_online.py, the 4over6 setting).  global_scale=(gs_w, 1/gs_w): use a
    weight scale shared with other tensors (see shared_scale_group) instead of
    this weight's own amax.
    """

    def __init__(self, weight: torch.Tensor, bias: torch.Tensor | None = None, per_token: bool = False,
                 four_over_six: bool = False, global_scale: tuple[torch.Tensor, torch.Tensor] | None = None):
        if weight.dim() != 2:
            raise ValueError(f"expects a 2-D weight, got shape {tuple(weight.shape)}")
        if weight.shape[1] % 16 != 0:
            raise ValueError(f"K must be a multiple of 16, got shape {tuple(weight.shape)}")
        w = coerce_input(weight).contiguous()
        self.out_features, self.in_features = w.shape
        self.per_token = per_token
        fmax = FP8_FP4_MAX_4OVER6 if four_over_six else FP8_FP4_MAX
        if global_scale is None and self.in_features % 64 == 0:
            self.weight, self.gs_w, self.inv_gs_w, _ = nvfp4_quantize_weight(w, fmax)
        else:
            if global_scale is None:
                self.gs_w, self.inv_gs_w = nvfp4_global_scale(amax(w), fmax)
            else:
                self.gs_w, self.inv_gs_w = global_scale
            self.weight = nvfp4_quantize(w, self.gs_w)
        self.gs_x = torch.ones(1, dtype=torch.float32, device=w.device)
        # per-token: the GEMM applies 1/gs_w here and 1/gs_x[m] as the row scale
        self.alpha = self.inv_gs_w if per_token else nvfp4_alpha(self.gs_x, self.gs_w)
        self.bias = None if bias is None else coerce_bf16(bias).contiguous()

    def quantize_input(self, x: torch.Tensor, sf_layout: str = "128x4") -> NVFP4Tensor:
        x = coerce_input(x)
        return nvfp4_quantize(x, None if self.per_token else self.gs_x, per_row=self.per_token, sf_layout=sf_layout)

    def rmsnorm_quantize_input(self, x: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-6) -> NVFP4Tensor:
        """RMSNorm(x) * gamma quantized for this layer in one kernel: pass the
        result as `pre_quantized` (the fused norm+quant producer)."""
        return nvfp4_rmsnorm_quantize(coerce_bf16(x), coerce_bf16(gamma).contiguous(), eps,
                                      None if self.per_token else self.gs_x, per_row=self.per_token)

    def layernorm_quantize_input(self, x: torch.Tensor, gamma: torch.Tensor | None = None,
                                 beta: torch.Tensor | None = None, eps: float = 1e-6) -> NVFP4Tensor:
        """LayerNorm(x) (* gamma + beta) quantized for this layer in one kernel:
        pass the result as `pre_quantized` (the fused norm+quant producer)."""
        g = None if gamma is None else coerce_bf16(gamma).contiguous()
        b = None if beta is None else coerce_bf16(beta).contiguous()
        return nvfp4_layernorm_quantize(coerce_bf16(x), g, b, eps, None if self.per_token else self.gs_x,
                                        per_row=self.per_token)

    def __call__(self, x: torch.Tensor, pre_quantized: NVFP4Tensor | None = None,
                 out_dtype: torch.dtype = torch.bfloat16, sf_layout: str = "128x4") -> torch.Tensor:
        """sf_layout "8x4": the activation's scales in 8-row tiles (mm_fp4's
        use_8x4_sf_layout), for at most 64 rows."""
        lead = x.shape[:-1]
        xq = pre_quantized if pre_quantized is not None else self.quantize_input(x, sf_layout)
        y = nvfp4_gemm(xq, self.weight, self.alpha, xq.row_inv_gs if self.per_token else None, self.bias,
                       out_dtype=out_dtype)
        return y.view(*lead, self.out_features)


    @classmethod
    def shared_scale_group(cls, weights, biases=None, per_token: bool = False, four_over_six: bool = False):
        """Linear layers whose weights share one global scale from their joint
        amax (the gated w1/w3 pair of nvfp4_online.py)."""
        ws = [coerce_input(w).contiguous() for w in weights]
        if not ws:
            raise ValueError("shared_scale_group needs at least one weight")
        a = amax(ws[0])
        for w in ws[1:]:
            amax_into(w, a)
        scale = nvfp4_global_scale(a, FP8_FP4_MAX_4OVER6 if four_over_six else FP8_FP4_MAX)
        biases = [None] * len(ws) if biases is None else list(biases)
        return [cls(w, b, per_token=per_token, global_scale=scale) for w, b in zip(ws, biases)]


class MXFP8Linear:
    """W8A8 MXFP8 linear layer (weight quantized once; activation per call)."""

    def __init__(self, weight: torch.Tensor, bias: torch.Tensor | None = None):
        if weight.dim() != 2 or weight.shape[1] % 32 != 0:
            raise ValueError(f"expects a 2-D weight with K % 32 == 0, got {tuple(weight.shape)}")
        w = coerce_bf16(weight).contiguous()
        self.out_features, self.in_features = w.shape
        self.weight = mxfp8_quantize(w)
        self.bias = None if bias is None else coerce_bf16(bias).contiguous()

    def __call__(self, x: torch.Tensor, out_dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
        lead = x.shape[:-1]
        xq = mxfp8_quantize(coerce_bf16(x))
        return mxfp8_gemm(xq, self.weight, None, self.bias, out_dtype=out_dtype).view(*lead, self.out_features)
