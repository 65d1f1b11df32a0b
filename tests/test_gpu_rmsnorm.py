"""Fused RMSNorm + NVFP4 quantize on the GPU vs the oracle's reading (the
producer of the pre-quantized activation of hao-ai-lab-FastVideo
nvfp4_config.py, NVFP4QuantizeMethod.apply).

The kernel's mean of squares has relative error <= 2^-24 (pairs of exact
squares added in fp32, pair sums in fp64 in any order, one rounding to fp32):
with the correctly rounded rsqrt after it, rstd lies within 0.5 ulp + 2^-24
relative of the true value, so within 2 fp32 ulp of the exactly rounded one,
which is the tolerance here.  Everything after it -- y in bf16, the group
scales and codes, per-token scales -- is checked bit for bit by running the
oracle from the rstd the kernel reports."""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_05_b200 import api
from block_scaled_precision_05_b200 import workloads as wl
from tests._gpu import DEV, assert_gemm_close, down, up_bf16

pytestmark = pytest.mark.gpu


def _case(M, K, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[rng.random((M, K)) < 0.001] *= 50
    g = (1.0 + 0.2 * rng.standard_normal(K)).astype(np.float32)
    return wl.f32_to_bf16_bits(x), wl.f32_to_bf16_bits(g)


def _ulps(a, b):
    return np.abs(a.view(np.int32).astype(np.int64) - b.view(np.int32).astype(np.int64))


# K = 1536 and 2048 take the register-resident kernel (ragged, exact-tile and
# multi-iteration row counts); the others the three-pass kernel.
SHAPES = [(1, 16), (7, 48), (130, 1536), (300, 5120), (64, 13824), (129, 80), (257, 1024), (1, 1536), (256, 2048),
          (4100, 1536), (129, 2048)]


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("per_row", [False, True])
def test_rmsnorm_quantize(M, K, per_row):
    x, g = _case(M, K, seed=M + 7 * K)
    eps = 1e-6
    rstd = torch.empty(M, dtype=torch.float32, device=DEV)
    gs = None if per_row else torch.tensor([0.75], dtype=torch.float32, device=DEV)
    q = api.nvfp4_rmsnorm_quantize(up_bf16(x), up_bf16(g), eps, gs, per_row=per_row, rstd_out=rstd)
    assert api.device_status() == 0
    r_gpu = down(rstd)
    r_exact = oracle.rmsnorm_rstd(x, eps)
    assert _ulps(r_gpu, r_exact).max() <= 2
    codes, sf, _, g_rows, inv_rows = oracle.rmsnorm_quantize(x, g, eps, np.float32(0.75), per_row=per_row,
                                                               rstd=r_gpu)
    assert np.array_equal(down(q.codes), codes)
    assert np.array_equal(down(q.sf), sf)
    if per_row:
        assert np.array_equal(down(q.row_gs), g_rows) and np.array_equal(down(q.row_inv_gs), inv_rows)


def test_equals_norm_then_quantize():
    """Same bytes as writing y = RMSNorm(x) in bf16 and quantizing it."""
    M, K = 300, 1536
    x, g = _case(M, K, seed=61)
    rstd = torch.empty(M, dtype=torch.float32, device=DEV)
    gs = torch.ones(1, dtype=torch.float32, device=DEV)
    fused = api.nvfp4_rmsnorm_quantize(up_bf16(x), up_bf16(g), 1e-6, gs, rstd_out=rstd)
    y = oracle.rmsnorm_bf16(x, g, down(rstd))
    plain = api.nvfp4_quantize(up_bf16(y), gs)
    assert torch.equal(fused.codes, plain.codes) and torch.equal(fused.sf, plain.sf)


def test_norm_quantized_linear():
    M, N, K = 256, 768, 1536
    x, g = _case(M, K, seed=62)
    W = wl.f32_to_bf16_bits((np.random.default_rng(63).standard_normal((N, K)) * 0.02).astype(np.float32))
    layer = api.NVFP4Linear(up_bf16(W))
    rstd = torch.empty(M, dtype=torch.float32, device=DEV)
    xq = api.nvfp4_rmsnorm_quantize(up_bf16(x), up_bf16(g), 1e-6, layer.gs_x, rstd_out=rstd)
    D = layer(up_bf16(x), pre_quantized=xq)
    assert api.device_status() == 0
    ca, sa, _, _, _ = oracle.rmsnorm_quantize(x, g, 1e-6, np.float32(1.0), rstd=down(rstd))
    gso = oracle.nvfp4_global_scale(oracle.amax_bf16(W))
    cb, sb = oracle.nvfp4_quantize(W, gso)
    ref, bound = oracle.linear_reference(oracle.nvfp4_dequantize(ca, sa, K), oracle.nvfp4_dequantize(cb, sb, K),
                                         alpha=np.float32(1) / (np.float32(1) * gso), row_scale=None, bias=None)
    assert_gemm_close(D, ref, bound, "rmsnorm-quantized linear")


@pytest.mark.parametrize("K", [1536, 2048, 1024])
def test_rmsnorm_strided_rows(K):
    """Rows read with a row stride larger than K (a column slice of a wider tensor)."""
    M = 200
    x, g = _case(M, K + 64, seed=K + 5)
    xs = up_bf16(x)[:, :K]
    assert xs.stride(0) == K + 64
    rstd = torch.empty(M, dtype=torch.float32, device=DEV)
    q = api.nvfp4_rmsnorm_quantize(xs, up_bf16(g[:K].copy()), 1e-6, None, per_row=True, rstd_out=rstd)
    assert api.device_status() == 0
    xk = np.ascontiguousarray(x[:, :K])
    r_gpu = down(rstd)
    assert _ulps(r_gpu, oracle.rmsnorm_rstd(xk, 1e-6)).max() <= 2
    codes, sf, _, g_rows, _ = oracle.rmsnorm_quantize(xk, g[:K].copy(), 1e-6, np.float32(1.0), per_row=True,
                                                      rstd=r_gpu)
    assert np.array_equal(down(q.codes), codes) and np.array_equal(down(q.sf), sf)
    assert np.array_equal(down(q.row_gs), g_rows)
