"""ctypes loader for libbsp.so, the C-ABI CUDA library (include/bsp.h).

Argument marshalling only.  There is no fallback: if the library is missing or
the device is not an sm_100 GPU, every call raises.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbsp.so")

BSP_OK = 0
BSP_ERR_INVALID_ARG = 1
BSP_ERR_ALIGNMENT = 2
BSP_ERR_UNSUPPORTED_DEVICE = 3
BSP_ERR_CUDA = 4
BSP_ERR_TIMEOUT = 5
BSP_SF_PER_TENSOR = 0
BSP_SF_PER_ROW = 1
BSP_OUT_BF16 = 0
BSP_OUT_F32 = 1
BSP_IN_BF16 = 0
BSP_IN_F16 = 1
BSP_SF_LAYOUT_128X4 = 0
BSP_SF_LAYOUT_8X4 = 1
BSP_NORM_RMS = 0
BSP_NORM_LAYER = 1

_vp, _i64, _i32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t

BSP_WEIGHT_BATCH_MAX = 256


class BspWeightDesc(ctypes.Structure):
    """bsp_weight_desc of include/bsp.h (one weight of nvfp4_quantize_weights)."""
    _fields_ = [("w", _vp), ("N", _i64), ("K", _i64), ("ld_w", _i64), ("amax", _vp), ("gs", _vp), ("inv_gs", _vp),
                ("codes", _vp), ("sf", _vp)]

# name -> (restype, argtypes), one entry per function declared in include/bsp.h
SIGNATURES = {
    "bsp_status_string": (ctypes.c_char_p, [_i32]),
    "bsp_version": (_i32, []),
    "bsp_nvfp4_sf_bytes": (_sz, [_i64, _i64]),
    "bsp_mxfp8_sf_bytes": (_sz, [_i64, _i64]),
    "bsp_nvfp4_sf_bytes_layout": (_sz, [_i64, _i64, _i32]),
    "bsp_amax_bf16": (_i32, [_vp, _i64, _vp, _vp]),
    "bsp_amax_bf16_into": (_i32, [_vp, _i64, _vp, _vp]),
    "bsp_amax_f16": (_i32, [_vp, _i64, _vp, _vp]),
    "bsp_amax_f16_into": (_i32, [_vp, _i64, _vp, _vp]),
    "bsp_nvfp4_global_scale": (_i32, [_vp, _vp, _vp, _vp]),
    "bsp_nvfp4_global_scale_max": (_i32, [_vp, ctypes.c_float, _vp, _vp, _vp]),
    "bsp_nvfp4_alpha": (_i32, [_vp, _vp, _vp, _vp]),
    "nvfp4_quantize_weight": (_i32, [_vp, _i32, _i64, _i64, _i64, ctypes.c_float, _vp, _vp, _vp, _vp, _vp, _vp, _i64,
                                     _vp]),
    "bsp_nvfp4_quantize_weight_workspace_bytes": (_i32, [_i32, _vp]),
    "nvfp4_quantize_weight_static": (_i32, [_vp, _i32, _i64, _i64, _i64, ctypes.c_float, _vp, _vp, _vp, _vp, _vp,
                                            _vp]),
    "nvfp4_quantize_weights": (_i32, [_vp, _i32, _i32, ctypes.c_float, _vp, _i64, _vp]),
    "nvfp4_quantize": (_i32, [_vp, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _vp, _vp, _vp]),
    "nvfp4_quantize_f16": (_i32, [_vp, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _vp, _vp, _vp]),
    "nvfp4_quantize_ex": (_i32, [_vp, _i32, _i64, _i64, _i64, _vp, _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "nvfp4_rmsnorm_quantize": (_i32, [_vp, _i64, _i64, _i64, _vp, ctypes.c_float, _vp, _i32, _vp, _vp, _vp, _vp, _vp,
                                      _vp]),
    "nvfp4_layernorm_quantize": (_i32, [_vp, _i64, _i64, _i64, _vp, _vp, ctypes.c_float, _vp, _i32, _vp, _vp, _vp,
                                        _vp, _vp, _vp, _vp]),
    "nvfp4_gemm": (_i32, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _i32, _i64, _vp]),
    "nvfp4_gemm_ex": (_i32, [_vp, _vp, _i32, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _i32, _i64, _vp]),
    "mxfp8_quantize": (_i32, [_vp, _i64, _i64, _i64, _vp, _vp, _vp]),
    "mxfp8_gemm": (_i32, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _i32, _i64, _vp]),
    "bsp_device_status": (_i32, [_vp]),
    "bsp_debug_encode_e2m1": (_i32, [_vp, _i64, _vp, _vp]),
    "bsp_debug_encode_e4m3": (_i32, [_vp, _i64, _vp, _vp]),
    "bsp_debug_wait_timeout": (_i32, [_i64, _vp]),
    "bsp_debug_norm_stats": (_i32, [_vp, _i64, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _vp]),
}


class BSPError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m block_scaled_precision_05_b200.csrc.build` (or __graft_entry__.build()). "
                "There is no fallback implementation.")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().bsp_status_string(int(status)).decode()


def check(status: int, what: str) -> None:
    if status != BSP_OK:
        raise BSPError(status, what)
