"""B200-native (sm_100a) block-scaled linear layers: W4A4 NVFP4 and W8A8 MXFP8.

The compute path is libbsp.so (C ABI, include/bsp.h): hand-written CUDA
quantize kernels and tcgen05 block-scaled GEMM kernels.  This package is the
thin PyTorch binding (device memory and streams only) plus the seeded
synthetic workloads used by the tests and the benchmark.
"""
from .api import (  # noqa: F401
    MXFP8Linear,
    MXFP8Tensor,
    NVFP4Linear,
    NVFP4Tensor,
    amax,
    coerce_input,
    device_status,
    mxfp8_gemm,
    mxfp8_quantize,
    mxfp8_sf_bytes,
    nvfp4_alpha,
    nvfp4_gemm,
    nvfp4_global_scale,
    nvfp4_layernorm_quantize,
    nvfp4_quantize,
    nvfp4_rmsnorm_quantize,
    nvfp4_sf_bytes,
)
from ._native import BSPError, LIB_PATH  # noqa: F401
