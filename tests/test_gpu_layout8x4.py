"""The 8x4 activation-scale layout on the GPU (hao-ai-lab-FastVideo
nvfp4_config.py: SfLayout.layout_8x4, mm_fp4's use_8x4_sf_layout): quantize
bit-exact against the oracle's 8x4 map, and the M <= 64 GEMM on 8x4 scales
bit-identical to the same GEMM on 128x4 scales (the tensor core receives the
same scale values) and within tolerance of the oracle."""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_05_b200 import _native as nat
from block_scaled_precision_05_b200 import api
from block_scaled_precision_05_b200 import workloads as wl
from tests._gpu import DEV, assert_gemm_close, down, up_bf16

pytestmark = pytest.mark.gpu


def _x(M, K, seed):
    return wl.f32_to_bf16_bits(np.random.default_rng(seed).standard_normal((M, K)).astype(np.float32))


@pytest.mark.parametrize("M", [1, 7, 8, 9, 16, 33, 64, 130])
@pytest.mark.parametrize("K", [64, 80, 1536, 5120])
@pytest.mark.parametrize("per_row", [False, True])
def test_quantize_8x4_bit_exact(M, K, per_row):
    x = _x(M, K, seed=M * 11 + K)
    if per_row:
        q = api.nvfp4_quantize(up_bf16(x), per_row=True, sf_layout="8x4")
        gs, _ = oracle.row_global_scales(x)
        codes, sf = oracle.nvfp4_quantize(x, gs, per_row=True, layout="8x4")
    else:
        q = api.nvfp4_quantize(up_bf16(x), torch.tensor([0.625], device=DEV), sf_layout="8x4")
        codes, sf = oracle.nvfp4_quantize(x, np.float32(0.625), layout="8x4")
    assert q.sf.numel() == oracle.sf_bytes(M, K // 16, "8x4")
    assert np.array_equal(down(q.codes), codes)
    assert np.array_equal(down(q.sf), sf)


@pytest.mark.parametrize("M", [1, 5, 16, 17, 40, 64])
@pytest.mark.parametrize("per_token", [False, True])
def test_gemm_8x4_equals_128x4(M, per_token):
    N, K = 1024, 5120
    A = _x(M, K, seed=M + 500)
    W = wl.f32_to_bf16_bits((np.random.default_rng(501).standard_normal((N, K)) * 0.02).astype(np.float32))
    bias = wl.f32_to_bf16_bits((np.random.default_rng(502).standard_normal(N) * 0.01).astype(np.float32))
    layer = api.NVFP4Linear(up_bf16(W), up_bf16(bias), per_token=per_token)
    x = up_bf16(A)
    D128 = layer(x)
    D8 = layer(x, sf_layout="8x4")
    assert api.device_status() == 0
    assert torch.equal(D8, D128)
    gso = oracle.nvfp4_global_scale(oracle.amax_bf16(W))
    cb, sb = oracle.nvfp4_quantize(W, gso)
    if per_token:
        gs_rows, inv_rows = oracle.row_global_scales(A)
        ca, sa = oracle.nvfp4_quantize(A, gs_rows, per_row=True, layout="8x4")
        alpha, rs = np.float32(1) / gso, inv_rows
    else:
        ca, sa = oracle.nvfp4_quantize(A, np.float32(1.0), layout="8x4")
        alpha, rs = np.float32(1) / (np.float32(1) * gso), None
    ref, bound = oracle.linear_reference(oracle.nvfp4_dequantize(ca, sa, K, layout="8x4"),
                                         oracle.nvfp4_dequantize(cb, sb, K), alpha=alpha, row_scale=rs, bias=bias)
    assert_gemm_close(D8, ref, bound, f"8x4 GEMM M={M}")


def test_8x4_rejected_above_64_rows():
    A = _x(65, 256, seed=7)
    W = _x(128, 256, seed=8)
    layer = api.NVFP4Linear(up_bf16(W))
    with pytest.raises(nat.BSPError):
        layer(up_bf16(A), sf_layout="8x4")
