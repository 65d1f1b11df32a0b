"""CPU oracle for the block-scaled (NVFP4 / MXFP8) linear layer.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  It shares no code with the CUDA library and never calls it.

The scalar, bit-exact parts (format decoders, round-to-nearest-even encoders,
the NVFP4 and MXFP8 group quantizers and the 128x4 scale-tile map) are plain C
in ``bsp_oracle.c``, compiled with gcc and no floating-point contraction.  The
contraction is a float64 matrix product of the decoded operands (numpy, a
library matmul used as one step):

    y[m, n] = alpha * row_scale[m] * sum_k decA[m, k] * decB[n, k] + bias[n]

which is the definition of the block-scaled GEMM the pages call
(``mm_fp4(x_fp4, w_fp4.T, x_scale, w_scale.T, 1/(gs_x*gs_w), bf16)`` followed by
``out + bias`` in hao-ai-lab-FastVideo nvfp4_qat_config.py,
``NVFP4QATQuantizeMethod.apply``; the MXFP8 product of vllm-omni
mxfp8_config.py, ``NPUMxfp8LinearMethod._quant_matmul``, with alpha = 1).

Parity pins for every function live in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor
from fractions import Fraction

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bsp_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

_lib = None


def build(force: bool = False) -> str:
    """Compile ``bsp_oracle.c`` into ``_build/liboracle.so`` (gcc)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        i64, f32, f64, i32 = ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_int
        vp = ctypes.c_void_p
        L.bspo_bf16_value.restype = f64
        L.bspo_bf16_value.argtypes = [ctypes.c_uint16]
        L.bspo_e2m1_value.restype = f64
        L.bspo_e2m1_value.argtypes = [i32]
        L.bspo_e4m3_value.restype = f64
        L.bspo_e4m3_value.argtypes = [i32]
        L.bspo_e8m0_value.restype = f64
        L.bspo_e8m0_value.argtypes = [i32]
        L.bspo_e2m1_encode.restype = i32
        L.bspo_e2m1_encode.argtypes = [f64]
        L.bspo_e4m3_encode.restype = i32
        L.bspo_e4m3_encode.argtypes = [f64]
        L.bspo_bf16_round.restype = ctypes.c_uint16
        L.bspo_bf16_round.argtypes = [f64]
        L.bspo_sf_offset.restype = i64
        L.bspo_sf_offset.argtypes = [i64, i64, i64]
        L.bspo_sf_bytes.restype = i64
        L.bspo_sf_bytes.argtypes = [i64, i64]
        L.bspo_sf_offset_8x4.restype = i64
        L.bspo_sf_offset_8x4.argtypes = [i64, i64, i64]
        L.bspo_sf_bytes_8x4.restype = i64
        L.bspo_sf_bytes_8x4.argtypes = [i64, i64]
        L.bspo_nvfp4_quantize_layout.restype = i32
        L.bspo_nvfp4_quantize_layout.argtypes = [vp, i64, i64, i64, i32, i32, vp, i32, vp, vp]
        L.bspo_nvfp4_dequantize_rows_layout.restype = None
        L.bspo_nvfp4_dequantize_rows_layout.argtypes = [vp, vp, i64, i32, vp, i64, vp]
        L.bspo_amax_bf16.restype = f32
        L.bspo_amax_bf16.argtypes = [vp, i64]
        L.bspo_nvfp4_global_scale.restype = f32
        L.bspo_nvfp4_global_scale.argtypes = [f32]
        L.bspo_nvfp4_global_scale_max.restype = f32
        L.bspo_nvfp4_global_scale_max.argtypes = [f32, f32]
        L.bspo_row_global_scales.restype = None
        L.bspo_row_global_scales.argtypes = [vp, i64, i64, i64, vp, vp]
        L.bspo_nvfp4_quantize_group.restype = None
        L.bspo_nvfp4_quantize_group.argtypes = [vp, f32, vp, vp]
        L.bspo_nvfp4_quantize.restype = i32
        L.bspo_nvfp4_quantize.argtypes = [vp, i64, i64, i64, vp, i32, vp, vp]
        L.bspo_nvfp4_quantize_fmt.restype = i32
        L.bspo_nvfp4_quantize_fmt.argtypes = [vp, i64, i64, i64, i32, vp, i32, vp, vp]
        L.bspo_f16_value.restype = ctypes.c_double
        L.bspo_f16_value.argtypes = [ctypes.c_uint16]
        L.bspo_amax_fmt.restype = f32
        L.bspo_amax_fmt.argtypes = [vp, i64, i32]
        L.bspo_row_global_scales_fmt.restype = None
        L.bspo_row_global_scales_fmt.argtypes = [vp, i64, i64, i64, i32, vp, vp]
        L.bspo_mxfp8_quantize_group.restype = None
        L.bspo_mxfp8_quantize_group.argtypes = [vp, vp, vp]
        L.bspo_mxfp8_quantize.restype = i32
        L.bspo_mxfp8_quantize.argtypes = [vp, i64, i64, i64, vp, vp]
        L.bspo_nvfp4_dequantize_rows.restype = None
        L.bspo_nvfp4_dequantize_rows.argtypes = [vp, vp, i64, vp, i64, vp]
        L.bspo_mxfp8_dequantize_rows.restype = None
        L.bspo_mxfp8_dequantize_rows.argtypes = [vp, vp, i64, vp, i64, vp]
        L.bspo_bf16_round_array.restype = None
        L.bspo_bf16_round_array.argtypes = [vp, i64, vp]
        L.bspo_e4m3_encode_array.restype = None
        L.bspo_e4m3_encode_array.argtypes = [vp, i64, vp]
        L.bspo_e2m1_encode_array.restype = None
        L.bspo_e2m1_encode_array.argtypes = [vp, i64, vp]
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _threads(threads):
    return max(1, threads if threads else (os.cpu_count() or 1))


# --------------------------------------------------------------------------- scalars
def bf16_value(bits: int) -> float:
    return lib().bspo_bf16_value(int(bits))


def e2m1_value(code: int) -> float:
    return lib().bspo_e2m1_value(int(code))


def e4m3_value(byte: int) -> float:
    return lib().bspo_e4m3_value(int(byte))


def e8m0_value(byte: int) -> float:
    return lib().bspo_e8m0_value(int(byte))


def e2m1_encode(v) -> np.ndarray:
    """e2m1 RNE-satfinite codes (0..15, sign in bit 3) of fp32 values; -1 for NaN."""
    a = np.ascontiguousarray(np.asarray(v, dtype=np.float32).reshape(-1))
    out = np.empty(a.size, dtype=np.int8)
    lib().bspo_e2m1_encode_array(_ptr(a), a.size, _ptr(out))
    return out.reshape(np.shape(v))


def e4m3_encode(v) -> np.ndarray:
    """e4m3fn RNE-satfinite bytes of fp32 values (NaN -> 0x7F)."""
    a = np.ascontiguousarray(np.asarray(v, dtype=np.float32).reshape(-1))
    out = np.empty(a.size, dtype=np.uint8)
    lib().bspo_e4m3_encode_array(_ptr(a), a.size, _ptr(out))
    return out.reshape(np.shape(v))


def bf16_round(y) -> np.ndarray:
    """Nearest-even bf16 bit patterns (uint16) of float64 values, rounded once."""
    a = np.ascontiguousarray(np.asarray(y, dtype=np.float64).reshape(-1))
    out = np.empty(a.size, dtype=np.uint16)
    lib().bspo_bf16_round_array(_ptr(a), a.size, _ptr(out))
    return out.reshape(np.shape(y))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact values of bf16 bit patterns (a bf16 is the top half of an fp32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


LAYOUTS = {"128x4": 0, "8x4": 1}


def sf_offset(r: int, c: int, cols_padded: int, layout: str = "128x4") -> int:
    if layout == "8x4":
        return lib().bspo_sf_offset_8x4(int(r), int(c), int(cols_padded))
    return lib().bspo_sf_offset(int(r), int(c), int(cols_padded))


def sf_bytes(rows: int, cols: int, layout: str = "128x4") -> int:
    """Bytes of a tile-mapped scale buffer for [rows, cols] scales."""
    if layout == "8x4":
        return lib().bspo_sf_bytes_8x4(int(rows), int(cols))
    return lib().bspo_sf_bytes(int(rows), int(cols))


# --------------------------------------------------------------------------- global scales
FORMATS = {"bf16": 0, "f16": 1}


def amax_bf16(x: np.ndarray) -> float:
    a = np.ascontiguousarray(x, dtype=np.uint16).reshape(-1)
    return float(np.float32(lib().bspo_amax_bf16(_ptr(a), a.size)))


def amax_f16(x: np.ndarray) -> float:
    """amax of fp16 bit patterns (NaN as 0, +-inf as 65504)."""
    a = np.ascontiguousarray(x, dtype=np.uint16).reshape(-1)
    return float(np.float32(lib().bspo_amax_fmt(_ptr(a), a.size, 1)))


def f16_value(bits: int) -> float:
    """Exact value of one fp16 bit pattern."""
    return float(lib().bspo_f16_value(int(bits)))


def nvfp4_global_scale(amax: float, fp8_fp4_max: float | None = None) -> np.float32:
    """gs = fp8_fp4_max / amax in fp32 (1 for amax 0); fp8_fp4_max defaults to 448*6."""
    if fp8_fp4_max is None:
        return np.float32(lib().bspo_nvfp4_global_scale(float(np.float32(amax))))
    return np.float32(lib().bspo_nvfp4_global_scale_max(float(np.float32(amax)), float(np.float32(fp8_fp4_max))))


def row_global_scales(x: np.ndarray, fmt: str = "bf16"):
    """Per-row (per-token) encode scales gs[m] and decode factors 1/gs[m] (fp32)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    M, K = x.shape
    gs = np.empty(M, np.float32)
    inv = np.empty(M, np.float32)
    lib().bspo_row_global_scales_fmt(_ptr(x), M, K, K, FORMATS[fmt], _ptr(gs), _ptr(inv))
    return gs, inv


# --------------------------------------------------------------------------- quantizers
def _row_chunks(M: int, threads: int):
    """Row ranges starting at multiples of 128, so each owns whole scale bands."""
    per = -(-M // max(1, threads))
    per = -(-per // 128) * 128
    return [(m0, min(M, m0 + per)) for m0 in range(0, M, per)]


def nvfp4_quantize(x: np.ndarray, gs, per_row: bool = False, threads: int | None = None, fmt: str = "bf16",
                   layout: str = "128x4"):
    """NVFP4 quantization of bf16 (or, fmt="f16", fp16) bit patterns ``x`` [M, K] along K.

    Returns (codes uint8 [M, K/2], sf uint8 [sf_bytes(M, K/16)] in the 128x4 map).
    ``gs`` is one fp32 encode scale, or one per row if ``per_row``.
    """
    x = np.ascontiguousarray(x, dtype=np.uint16)
    M, K = x.shape
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    g = np.ascontiguousarray(np.asarray(gs, dtype=np.float32).reshape(-1))
    if per_row and g.size != M:
        raise ValueError("per-row scales need one value per row")
    codes = np.empty((M, K // 2), np.uint8)
    cols = K // 16
    cols_p = -(-cols // 4) * 4
    sf = np.empty(sf_bytes(M, cols, layout), np.uint8)
    if M == 0:
        return codes, sf
    L = lib()

    def run(rng):
        m0, m1 = rng
        gp = _ptr(g) + (4 * m0 if per_row else 0)
        # chunks start at multiples of 128 rows: whole 128-row bands, or 16 8-row tiles
        rc = L.bspo_nvfp4_quantize_layout(_ptr(x) + 2 * m0 * K, m1 - m0, K, K, FORMATS[fmt], LAYOUTS[layout], gp,
                                          int(per_row), _ptr(codes) + m0 * (K // 2), _ptr(sf) + m0 * cols_p)
        assert rc == 0

    chunks = _row_chunks(M, _threads(threads))
    with ThreadPoolExecutor(len(chunks)) as ex:
        list(ex.map(run, chunks))
    return codes, sf


def mxfp8_quantize(x: np.ndarray, threads: int | None = None):
    """MXFP8 quantization of bf16 bit patterns ``x`` [M, K] (groups of 32 along K).

    Returns (q uint8 e4m3 [M, K], sf uint8 e8m0 [sf_bytes(M, K/32)] in the 128x4 map).
    """
    x = np.ascontiguousarray(x, dtype=np.uint16)
    M, K = x.shape
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    q = np.empty((M, K), np.uint8)
    cols = K // 32
    cols_p = -(-cols // 4) * 4
    sf = np.empty(sf_bytes(M, cols), np.uint8)
    if M == 0:
        return q, sf
    L = lib()

    def run(rng):
        m0, m1 = rng
        rc = L.bspo_mxfp8_quantize(_ptr(x) + 2 * m0 * K, m1 - m0, K, K,
                                   _ptr(q) + m0 * K, _ptr(sf) + m0 * cols_p)
        assert rc == 0

    chunks = _row_chunks(M, _threads(threads))
    with ThreadPoolExecutor(len(chunks)) as ex:
        list(ex.map(run, chunks))
    return q, sf


# --------------------------------------------------------------------------- decoders
def _dequant(fn, codes, sf, K, rows, threads):
    rows = np.ascontiguousarray(np.arange(codes.shape[0]) if rows is None else rows, dtype=np.int64)
    out = np.empty((rows.size, K), np.float64)
    if rows.size == 0:
        return out
    codes = np.ascontiguousarray(codes)
    sf = np.ascontiguousarray(sf)
    n = _threads(threads)
    parts = np.array_split(np.arange(rows.size), min(n, rows.size))

    def run(idx):
        i0 = int(idx[0])
        fn(_ptr(codes), _ptr(sf), K, _ptr(rows) + 8 * i0, idx.size, _ptr(out) + 8 * K * i0)

    with ThreadPoolExecutor(len(parts)) as ex:
        list(ex.map(run, parts))
    return out


def nvfp4_dequantize(codes: np.ndarray, sf: np.ndarray, K: int, rows=None, threads=None,
                     layout: str = "128x4") -> np.ndarray:
    """Real values e2m1(code) * e4m3(scale) of the chosen rows, float64 [len(rows), K]."""
    if layout == "8x4":
        f = lib().bspo_nvfp4_dequantize_rows_layout
        return _dequant(lambda c, s, k, r, n, o: f(c, s, k, 1, r, n, o), codes, sf, K, rows, threads)
    return _dequant(lib().bspo_nvfp4_dequantize_rows, codes, sf, K, rows, threads)


def mxfp8_dequantize(q: np.ndarray, sf: np.ndarray, K: int, rows=None, threads=None) -> np.ndarray:
    """Real values e4m3(q) * e8m0(scale) of the chosen rows, float64 [len(rows), K]."""
    return _dequant(lib().bspo_mxfp8_dequantize_rows, q, sf, K, rows, threads)


# --------------------------------------------------------------------------- contraction
def linear_reference(decA: np.ndarray, decB: np.ndarray, alpha: float = 1.0,
                     row_scale=None, bias=None):
    """y = alpha * row_scale[m] * (decA @ decB.T) + bias[n] in float64.

    Returns (y, bound) where bound[m, n] = |alpha * row_scale[m]| * sum_k |decA * decB|,
    the scale of the accumulation-error tolerance.
    """
    acc = decA @ decB.T
    mag = np.abs(decA) @ np.abs(decB).T
    f = np.float64(np.float32(alpha))
    if row_scale is not None:
        f = f * np.asarray(row_scale, dtype=np.float32).astype(np.float64)[:, None]
    y = f * acc
    if bias is not None:
        y = y + bf16_bits_to_f64(bias)[None, :]
    return y, np.abs(f) * mag


# --------------------------------------------------------------------------- RMSNorm before the quantizer
# The producer of a pre-quantized activation (hao-ai-lab-FastVideo
# nvfp4_config.py, NVFP4QuantizeMethod.apply: `pre_quantized` from "fused
# norm+quant" calls).  The pages do not print the norm; the reading is RMSNorm
# with a weight, its output rounded to bf16 and then quantized as any bf16
# activation:
#   ms   = (1/K) sum_k x_k^2            (exact, then rounded once to fp32)
#   rstd = RN32(1 / sqrt(RN32(ms + eps)))
#   y_k  = bf16(RN32(RN32(x_k * rstd) * gamma_k))
def _rn_f32_ratio(p: int, q: int) -> np.float32:
    """The fp32 nearest to p/q (p >= 0, q > 0 integers), ties to even."""
    if p == 0:
        return np.float32(0.0)
    # e = floor(log2(p/q))
    e = p.bit_length() - q.bit_length()
    if (p << max(0, -e)) < (q << max(0, e)):
        e -= 1
    if e > 127:
        return np.float32(np.inf)
    shift = 23 - max(e, -126)  # fraction bits kept: 24 for normals, fewer below 2^-126
    num, den = (p << shift, q) if shift >= 0 else (p, q << -shift)
    n, rem = divmod(num, den)
    if 2 * rem > den or (2 * rem == den and (n & 1)):
        n += 1
    return np.float32(math.ldexp(float(n), -shift))  # n < 2^25: exact in fp64 and fp32


def _rsqrt_rn32(t: np.float32) -> np.float32:
    """RN32(1/sqrt(t)) for an fp32 t >= 0, decided exactly (IEEE: +0 for
    t = +inf, +inf for t = 0)."""
    if np.isinf(t):
        return np.float32(0.0)
    if t == 0:
        return np.float32(np.inf)
    tf = Fraction(float(t))
    c = np.float32(1.0 / math.sqrt(float(t)))
    for _ in range(4):  # the fp64 estimate is within an fp32 ulp: at most one step either way
        up = np.nextafter(c, np.float32(np.inf), dtype=np.float32)
        dn = np.nextafter(c, np.float32(0), dtype=np.float32)
        mid_up = (Fraction(float(c)) + Fraction(float(up))) / 2
        mid_dn = (Fraction(float(c)) + Fraction(float(dn))) / 2
        # z = t^(-1/2) > m  <=>  m^2 t < 1
        if mid_up * mid_up * tf < 1 or (mid_up * mid_up * tf == 1 and (np.float32(up).view(np.uint32) & 1) == 0):
            c = up
        elif mid_dn * mid_dn * tf > 1 or (mid_dn * mid_dn * tf == 1 and (np.float32(dn).view(np.uint32) & 1) == 0):
            c = dn
        else:
            return c
    raise AssertionError("rsqrt rounding did not settle")


def _bf16_exact_parts(bits: np.ndarray):
    """(m, e) integers with value = m * 2^e for each bf16 pattern (finite)."""
    b = np.asarray(bits, dtype=np.int64)
    sign = np.where(b & 0x8000, -1, 1)
    ex = (b >> 7) & 0xFF
    man = b & 0x7F
    m = np.where(ex == 0, man, man | 0x80) * sign
    e = np.where(ex == 0, -133, ex - 134)
    return m, e


def rmsnorm_rstd(x: np.ndarray, eps: float) -> np.ndarray:
    """Exact-reading rstd per row of bf16 bit patterns x [M, K] (fp32 [M])."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    M, K = x.shape
    out = np.empty(M, np.float32)
    e32 = np.float32(eps)
    for r in range(M):
        m, e = _bf16_exact_parts(x[r])
        emin = int(e.min())
        s = 0
        for mi, ei in zip(m.tolist(), e.tolist()):
            s += (mi * mi) << (2 * (ei - emin))
        # ms = s * 2^(2 emin) / K
        if 2 * emin >= 0:
            ms = _rn_f32_ratio(s << (2 * emin), K)
        else:
            ms = _rn_f32_ratio(s, K << (-2 * emin))
        t = np.float32(ms + e32)  # fp32 add, round to nearest even
        out[r] = _rsqrt_rn32(t)
    return out


def rmsnorm_bf16(x: np.ndarray, gamma: np.ndarray, rstd: np.ndarray) -> np.ndarray:
    """y = bf16(RN32(RN32(x * rstd) * gamma)) as bf16 bit patterns [M, K]."""
    xv = bf16_bits_to_f64(x).astype(np.float32)  # exact
    gv = bf16_bits_to_f64(gamma).astype(np.float32)
    y = (xv * np.asarray(rstd, np.float32)[:, None]) * gv[None, :]  # two fp32 multiplies, each rounded
    return bf16_round(y.astype(np.float64))


def rmsnorm_quantize(x: np.ndarray, gamma: np.ndarray, eps: float, gs=None, per_row: bool = False):
    """RMSNorm to bf16, then NVFP4 quantization.
    Returns (codes, sf, rstd, row_gs or None, row_inv or None)."""
    rstd = rmsnorm_rstd(x, eps)
    y = rmsnorm_bf16(x, gamma, rstd)
    if per_row:
        g, inv = row_global_scales(y)
        codes, sf = nvfp4_quantize(y, g, per_row=True)
        return codes, sf, rstd, g, inv
    codes, sf = nvfp4_quantize(y, gs)
    return codes, sf, rstd, None, None


# --------------------------------------------------------------------------- LayerNorm before the quantizer
# The same producer with the norm of the Wan-2.1 blocks whose projections the
# pages quantize (hao-ai-lab-FastVideo nvfp4_qat_config.py, DEFAULT_FP4_LAYERS;
# nvfp4_config.py names the fused norm+quant call, not its norm).  Reading:
#   mean = (1/K) sum_k x_k                      (exact, then rounded once to fp32)
#   var  = (1/K) sum_k (x_k - mean_exact)^2     (exact population variance, rounded once)
#   rstd = RN32(1 / sqrt(RN32(var + eps)))
#   y_k  = bf16(RN32(RN32(RN32(RN32(x_k - mean) * rstd) * gamma_k) + beta_k))
# gamma and beta are optional; without them their steps are left out.
def _rn_f32_signed_ratio(p: int, q: int) -> np.float32:
    """The fp32 nearest to p/q for an integer p of either sign (q > 0), ties to
    even; a negative ratio that rounds to zero gives -0."""
    r = _rn_f32_ratio(abs(p), q)
    return np.float32(-r) if p < 0 else r


def layernorm_moments(x: np.ndarray):
    """(mean, var) per row of bf16 bit patterns x [M, K], each the exact value
    rounded once to fp32 (fp32 [M] each)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    M, K = x.shape
    mean = np.empty(M, np.float32)
    var = np.empty(M, np.float32)
    for r in range(M):
        m, e = _bf16_exact_parts(x[r])
        emin = int(e.min())
        s1 = 0
        s2 = 0
        for mi, ei in zip(m.tolist(), e.tolist()):
            s1 += mi << (ei - emin)
            s2 += (mi * mi) << (2 * (ei - emin))
        # sum x = s1 * 2^emin,  sum x^2 = s2 * 2^(2 emin)
        # mean = s1 * 2^emin / K;  var = (K s2 - s1^2) * 2^(2 emin) / K^2
        n = K * s2 - s1 * s1
        if emin >= 0:
            mean[r] = _rn_f32_signed_ratio(s1 << emin, K)
            var[r] = _rn_f32_ratio(n << (2 * emin), K * K)
        else:
            mean[r] = _rn_f32_signed_ratio(s1, K << -emin)
            var[r] = _rn_f32_ratio(n, (K * K) << (-2 * emin))
    return mean, var


def layernorm_stats(x: np.ndarray, eps: float):
    """(mean, rstd) per row (fp32 [M] each): the exact-reading mean and
    rstd = RN32(1/sqrt(RN32(var + eps)))."""
    mean, var = layernorm_moments(x)
    e32 = np.float32(eps)
    rstd = np.array([_rsqrt_rn32(np.float32(v + e32)) for v in var], np.float32)
    return mean, rstd


def layernorm_bf16(x: np.ndarray, gamma, beta, mean: np.ndarray, rstd: np.ndarray) -> np.ndarray:
    """y = bf16(RN32(RN32(RN32(RN32(x - mean) * rstd) * gamma) + beta)) as bf16
    bit patterns [M, K]; gamma / beta None leave their steps out."""
    xv = bf16_bits_to_f64(x).astype(np.float32)  # exact
    d = xv - np.asarray(mean, np.float32)[:, None]  # fp32 subtraction, rounded
    y = d * np.asarray(rstd, np.float32)[:, None]  # fp32 product, rounded
    if gamma is not None:
        y = y * bf16_bits_to_f64(gamma).astype(np.float32)[None, :]
    if beta is not None:
        y = y + bf16_bits_to_f64(beta).astype(np.float32)[None, :]
    return bf16_round(y.astype(np.float64))


def layernorm_quantize(x: np.ndarray, gamma, beta, eps: float, gs=None, per_row: bool = False):
    """LayerNorm to bf16, then NVFP4 quantization.
    Returns (codes, sf, mean, rstd, row_gs or None, row_inv or None)."""
    mean, rstd = layernorm_stats(x, eps)
    y = layernorm_bf16(x, gamma, beta, mean, rstd)
    if per_row:
        g, inv = row_global_scales(y)
        codes, sf = nvfp4_quantize(y, g, per_row=True)
        return codes, sf, mean, rstd, g, inv
    codes, sf = nvfp4_quantize(y, gs)
    return codes, sf, mean, rstd, None, None
