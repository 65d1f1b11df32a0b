"""The C-ABI library loads, exports every function include/bsp.h declares, and
rejects bad arguments on the host (no GPU needed: validation happens before any
device call)."""
import ctypes
import os
import re

import pytest

from block_scaled_precision_05_b200 import _native as nat

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "bsp.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", src)) - {"if", "sizeof"})


def test_header_and_binding_agree():
    assert sorted(nat.SIGNATURES) == _declared_functions()


def test_library_exports_every_declared_symbol():
    L = nat.lib()
    for name in _declared_functions():
        assert hasattr(L, name), name


def test_status_strings():
    for s in range(6):
        assert nat.status_string(s).startswith("BSP_")
    assert "UNKNOWN" in nat.status_string(99)
    assert nat.lib().bsp_version() >= 100


def test_sf_bytes_8x4():
    L = nat.lib()
    assert L.bsp_nvfp4_sf_bytes_layout(1, 64, nat.BSP_SF_LAYOUT_8X4) == 8 * 4
    assert L.bsp_nvfp4_sf_bytes_layout(9, 80, nat.BSP_SF_LAYOUT_8X4) == 16 * 8
    assert L.bsp_nvfp4_sf_bytes_layout(9, 80, nat.BSP_SF_LAYOUT_128X4) == L.bsp_nvfp4_sf_bytes(9, 80)
    assert L.bsp_nvfp4_sf_bytes_layout(9, 80, 5) == 0


@pytest.mark.parametrize("rows,K,nv,mx", [(1, 16, 512, 0), (128, 256, 128 * 16, 128 * 8), (129, 64, 256 * 4, 256 * 4),
                                          (32760, 5120, 32768 * 320, 32768 * 160), (0, 32, 0, 0), (5, 24, 0, 0)])
def test_sf_bytes(rows, K, nv, mx):
    import oracle
    assert nat.lib().bsp_nvfp4_sf_bytes(rows, K) == nv
    assert nat.lib().bsp_mxfp8_sf_bytes(rows, K) == mx
    if K % 16 == 0:
        assert nv == oracle.sf_bytes(rows, K // 16)


def test_host_validation_rejects_bad_arguments():
    L = nat.lib()
    p = ctypes.c_void_p(0x10000)  # never dereferenced: validation fails first
    odd = ctypes.c_void_p(0x10008)
    assert L.nvfp4_quantize(p, 4, 24, 24, p, 0, None, None, p, p, None) == nat.BSP_ERR_INVALID_ARG  # K % 16
    assert L.nvfp4_quantize(p, 4, 32, 16, p, 0, None, None, p, p, None) == nat.BSP_ERR_INVALID_ARG  # ld < K
    assert L.nvfp4_quantize(p, 4, 32, 32, p, 7, None, None, p, p, None) == nat.BSP_ERR_INVALID_ARG  # mode
    assert L.nvfp4_quantize(p, 4, 32, 32, None, 0, None, None, p, p, None) == nat.BSP_ERR_INVALID_ARG  # no gs
    assert L.nvfp4_quantize(odd, 4, 32, 32, p, 0, None, None, p, p, None) == nat.BSP_ERR_ALIGNMENT
    assert L.nvfp4_quantize(p, 0, 32, 32, p, 0, None, None, p, p, None) == nat.BSP_OK  # empty is a no-op
    assert L.mxfp8_quantize(p, 4, 48, 48, p, p, None) == nat.BSP_ERR_INVALID_ARG
    assert L.nvfp4_gemm(p, p, p, p, 4, 8, 48, None, None, None, p, 0, 8, None) == nat.BSP_ERR_INVALID_ARG  # K%32
    assert L.nvfp4_gemm(p, p, p, p, 4, 12, 64, None, None, None, p, 0, 12, None) == nat.BSP_ERR_INVALID_ARG  # N%8
    assert L.nvfp4_gemm(p, p, p, p, 4, 8, 64, None, None, None, p, 5, 8, None) == nat.BSP_ERR_INVALID_ARG  # dtype
    assert L.nvfp4_gemm(p, p, p, p, 4, 8, 64, None, None, None, odd, 0, 8, None) == nat.BSP_ERR_ALIGNMENT
    assert L.nvfp4_gemm(p, p, p, p, 4, 8, 64, None, None, None, p, 0, 12, None) == nat.BSP_ERR_ALIGNMENT  # ld_d
    assert L.nvfp4_gemm(p, p, p, p, 0, 8, 64, None, None, None, p, 0, 8, None) == nat.BSP_OK
    assert L.mxfp8_gemm(p, p, p, p, 4, 8, 48, None, None, p, 0, 8, None) == nat.BSP_ERR_INVALID_ARG
    assert L.bsp_amax_bf16(p, -1, p, None) == nat.BSP_ERR_INVALID_ARG
    assert L.bsp_amax_bf16_into(p, -1, p, None) == nat.BSP_ERR_INVALID_ARG
    assert L.nvfp4_quantize_ex(p, 2, 4, 32, 32, p, 0, 0, None, None, p, p, None) == nat.BSP_ERR_INVALID_ARG  # dtype
    assert L.nvfp4_quantize_ex(p, 0, 4, 32, 32, p, 0, 9, None, None, p, p, None) == nat.BSP_ERR_INVALID_ARG  # layout
    assert L.nvfp4_gemm_ex(p, p, 1, p, p, 65, 8, 64, None, None, None, p, 0, 8, None) == nat.BSP_ERR_INVALID_ARG  # 8x4 M>64
    assert L.nvfp4_gemm_ex(p, p, 7, p, p, 4, 8, 64, None, None, None, p, 0, 8, None) == nat.BSP_ERR_INVALID_ARG  # layout
    for bad in (-1.0, float("inf"), float("nan")):  # eps
        assert L.nvfp4_rmsnorm_quantize(p, 4, 32, 32, p, bad, p, 0, None, None, None, p, p, None) == \
            nat.BSP_ERR_INVALID_ARG
    assert L.nvfp4_rmsnorm_quantize(p, 4, 24, 24, p, 0.0, p, 0, None, None, None, p, p, None) == \
        nat.BSP_ERR_INVALID_ARG  # K % 16
    assert L.nvfp4_rmsnorm_quantize(p, 4, 32, 32, None, 0.0, p, 0, None, None, None, p, p, None) == \
        nat.BSP_ERR_INVALID_ARG  # no gamma
    assert L.nvfp4_rmsnorm_quantize(p, 4, (1 << 20) + 16, (1 << 20) + 16, p, 0.0, p, 0, None, None, None, p, p,
                                    None) == nat.BSP_ERR_INVALID_ARG  # K above the exact path's limit
    ln = L.nvfp4_layernorm_quantize
    for bad in (-1.0, float("inf"), float("nan")):  # eps
        assert ln(p, 4, 32, 32, None, None, bad, p, 0, None, None, None, None, p, p, None) == nat.BSP_ERR_INVALID_ARG
    assert ln(p, 4, 24, 24, None, None, 0.0, p, 0, None, None, None, None, p, p, None) == nat.BSP_ERR_INVALID_ARG
    assert ln(p, 4, 32784, 32784, None, None, 0.0, p, 0, None, None, None, None, p, p, None) == \
        nat.BSP_ERR_INVALID_ARG  # K > 32768
    assert ln(p, 4, 32, 32, None, None, 0.0, None, 0, None, None, None, None, p, p, None) == \
        nat.BSP_ERR_INVALID_ARG  # per-tensor without a global scale
    assert ln(p, 4, 32, 32, odd, None, 0.0, p, 0, None, None, None, None, p, p, None) == nat.BSP_ERR_ALIGNMENT
    assert ln(p, 4, 32, 32, None, odd, 0.0, p, 0, None, None, None, None, p, p, None) == nat.BSP_ERR_ALIGNMENT
    assert ln(p, 0, 32, 32, None, None, 0.0, p, 0, None, None, None, None, p, p, None) == nat.BSP_OK
    ns = L.bsp_debug_norm_stats
    assert ns(p, 4, 32, 32, 2, 0, p, p, None, None) == nat.BSP_ERR_INVALID_ARG  # norm
    assert ns(p, 4, 32, 32, nat.BSP_NORM_LAYER, 0, p, None, None, None) == nat.BSP_ERR_INVALID_ARG  # no var out
    assert ns(p, 4, 40, 40, nat.BSP_NORM_RMS, 0, p, None, None, None) == nat.BSP_ERR_INVALID_ARG  # K % 16
    for bad in (0.0, -2688.0, float("inf"), float("nan")):
        assert L.bsp_nvfp4_global_scale_max(p, bad, p, p, None) == nat.BSP_ERR_INVALID_ARG
    assert L.bsp_nvfp4_global_scale_max(p, 1536.0, None, None, None) == nat.BSP_ERR_INVALID_ARG
    assert L.bsp_debug_wait_timeout(10, None) == nat.BSP_ERR_INVALID_ARG
    qw = L.nvfp4_quantize_weight
    assert qw(p, 0, 4, 48, 48, 2688.0, None, p, p, p, p, p, 1 << 20, None) == nat.BSP_ERR_INVALID_ARG  # K % 64
    assert qw(p, 0, 4, 64, 32, 2688.0, None, p, p, p, p, p, 1 << 20, None) == nat.BSP_ERR_INVALID_ARG  # ld < K
    assert qw(p, 2, 4, 64, 64, 2688.0, None, p, p, p, p, p, 1 << 20, None) == nat.BSP_ERR_INVALID_ARG  # dtype
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        assert qw(p, 0, 4, 64, 64, bad, None, p, p, p, p, p, 1 << 20, None) == nat.BSP_ERR_INVALID_ARG
    assert qw(p, 0, 4, 64, 64, 2688.0, None, p, p, p, p, None, 1 << 20, None) == nat.BSP_ERR_INVALID_ARG  # no ws
    assert qw(p, 0, 4, 64, 64, 2688.0, None, None, p, p, p, p, 1 << 20, None) == nat.BSP_ERR_INVALID_ARG  # no gs
    assert qw(odd, 0, 4, 64, 64, 2688.0, None, p, p, p, p, p, 1 << 20, None) == nat.BSP_ERR_ALIGNMENT
    assert qw(p, 0, 4, 64, 68, 2688.0, None, p, p, p, p, p, 1 << 20, None) == nat.BSP_ERR_ALIGNMENT  # ld % 8
    assert L.bsp_nvfp4_quantize_weight_workspace_bytes(0, None) == nat.BSP_ERR_INVALID_ARG
    assert L.bsp_nvfp4_quantize_weight_workspace_bytes(5, p) == nat.BSP_ERR_INVALID_ARG
    qb = L.nvfp4_quantize_weights
    descs = (nat.BspWeightDesc * 2)()
    for d in descs:
        d.w, d.N, d.K, d.ld_w, d.gs, d.inv_gs, d.codes, d.sf = 0x10000, 4, 64, 64, 0x10000, 0x10000, 0x10000, 0x10000
    da = ctypes.addressof(descs)
    assert qb(da, nat.BSP_WEIGHT_BATCH_MAX + 1, 0, 2688.0, p, 1 << 20, None) == nat.BSP_ERR_INVALID_ARG  # count
    assert qb(da, -1, 0, 2688.0, p, 1 << 20, None) == nat.BSP_ERR_INVALID_ARG
    assert qb(None, 2, 0, 2688.0, p, 1 << 20, None) == nat.BSP_ERR_INVALID_ARG
    assert qb(da, 2, 2, 2688.0, p, 1 << 20, None) == nat.BSP_ERR_INVALID_ARG  # dtype
    assert qb(da, 2, 0, 0.0, p, 1 << 20, None) == nat.BSP_ERR_INVALID_ARG
    assert qb(da, 2, 0, 2688.0, None, 1 << 20, None) == nat.BSP_ERR_INVALID_ARG  # no workspace
    assert qb(da, 0, 0, 2688.0, p, 1 << 20, None) == nat.BSP_OK  # empty batch: nothing launched
    descs[1].K = 48
    assert qb(da, 2, 0, 2688.0, p, 1 << 20, None) == nat.BSP_ERR_INVALID_ARG  # K % 64 of the second weight
    descs[1].K, descs[1].w = 64, 0x10008
    assert qb(da, 2, 0, 2688.0, p, 1 << 20, None) == nat.BSP_ERR_ALIGNMENT
    qs = L.nvfp4_quantize_weight_static
    assert qs(p, 0, 4, 48, 48, 2688.0, None, p, p, p, p, None) == nat.BSP_ERR_INVALID_ARG  # K % 64
    assert qs(p, 3, 4, 64, 64, 2688.0, None, p, p, p, p, None) == nat.BSP_ERR_INVALID_ARG  # dtype
    assert qs(p, 0, 4, 64, 64, float("inf"), None, p, p, p, p, None) == nat.BSP_ERR_INVALID_ARG
    assert qs(p, 0, 4, 64, 64, 2688.0, None, None, p, p, p, None) == nat.BSP_ERR_INVALID_ARG  # no gs


def test_no_gpu_means_an_error_not_a_fallback():
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    L = nat.lib()
    p = ctypes.c_void_p(0x10000)
    st = L.nvfp4_quantize(p, 4, 32, 32, p, 0, None, None, p, p, None)
    assert st in (nat.BSP_ERR_CUDA, nat.BSP_ERR_UNSUPPORTED_DEVICE)


def test_weight_descriptor_layout():
    """The ctypes mirror of bsp_weight_desc has the header's layout (nine
    8-byte fields in declaration order, 72 bytes, no padding)."""
    names = ["w", "N", "K", "ld_w", "amax", "gs", "inv_gs", "codes", "sf"]
    assert [f[0] for f in nat.BspWeightDesc._fields_] == names
    assert ctypes.sizeof(nat.BspWeightDesc) == 72
    for i, n in enumerate(names):
        assert getattr(nat.BspWeightDesc, n).offset == 8 * i
    src = open(HEADER).read()
    assert "#define BSP_WEIGHT_BATCH_MAX 256" in src and nat.BSP_WEIGHT_BATCH_MAX == 256
