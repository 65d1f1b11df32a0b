"""Fused RMSNorm + NVFP4 quantize on the GPU against the oracle alone (the
producer of the pre-quantized activation of hao-ai-lab-FastVideo
nvfp4_config.py, NVFP4QuantizeMethod.apply).

The kernel's mean of squares is the exact mean rounded once to fp32 -- an fp64
sum with a proven error bound decides the rounding, exact integer sums decide
the rows it cannot -- so rstd, y, the group scales and codes and the per-token
scales all equal the oracle's bit for bit, with no value taken from the
kernel."""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_05_b200 import api
from block_scaled_precision_05_b200 import workloads as wl
from tests._gpu import DEV, assert_gemm_close, down, sample_bands, up_bf16

pytestmark = pytest.mark.gpu


def _case(M, K, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[rng.random((M, K)) < 0.001] *= 50
    g = (1.0 + 0.2 * rng.standard_normal(K)).astype(np.float32)
    return wl.f32_to_bf16_bits(x), wl.f32_to_bf16_bits(g)


def _check(q, rstd, x, g, eps, per_row, gs=np.float32(0.75)):
    codes, sf, r_ref, g_rows, inv_rows = oracle.rmsnorm_quantize(x, g, eps, gs, per_row=per_row)
    assert np.array_equal(down(rstd).view(np.uint32), r_ref.view(np.uint32))
    assert np.array_equal(down(q.codes), codes)
    assert np.array_equal(down(q.sf), sf)
    if per_row:
        assert np.array_equal(down(q.row_gs).view(np.uint32), g_rows.view(np.uint32))
        assert np.array_equal(down(q.row_inv_gs).view(np.uint32), inv_rows.view(np.uint32))


# K = 1536 and 2048 take the register-resident kernel (ragged, exact-tile and
# multi-iteration row counts); the others the multi-pass kernel.
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
    _check(q, rstd, x, g, eps, per_row)


def _midpoint_rows(K, n, seed):
    """Rows whose mean of squares is exactly halfway between two fp32 values
    (K/4 elements +-2, K/16 elements +-2^-10: mean 1 + 2^-24), scaled by
    powers of 4, shuffled, and variants just above and below the tie: the fp64
    bound cannot decide them, so the exact sums do."""
    rng = np.random.default_rng(seed)
    rows = []
    for i in range(n):
        r = np.zeros(K, np.float32)
        r[: K // 4] = 2.0
        r[K // 4: K // 4 + K // 16] = 2.0 ** -10
        if i % 3 == 1:
            r[-1] = 2.0 ** -40          # just above the tie
        elif i % 3 == 2:
            r[K // 4] = np.float32(2.0 ** -10 * (1 - 2.0 ** -8))  # just below
        r *= np.float32(2.0 ** rng.integers(-20, 20))
        r *= np.where(rng.random(K) < 0.5, -1.0, 1.0).astype(np.float32)
        rows.append(rng.permutation(r))
    return wl.f32_to_bf16_bits(np.stack(rows))


@pytest.mark.parametrize("K", [48, 1536, 2048, 5120])
@pytest.mark.parametrize("per_row", [False, True])
def test_rows_at_rounding_ties_take_the_exact_path(K, per_row):
    rand, g = _case(40, K, seed=K + 3)
    x = np.concatenate([_midpoint_rows(K, 24, seed=K), rand])
    M = x.shape[0]
    (ms,), path = api.norm_stats(up_bf16(x), "rms")
    assert (down(path)[:24:3] == 1).all()  # the exact ties cannot be settled by the fp64 bound
    rstd = torch.empty(M, dtype=torch.float32, device=DEV)
    gs = None if per_row else torch.tensor([0.75], dtype=torch.float32, device=DEV)
    q = api.nvfp4_rmsnorm_quantize(up_bf16(x), up_bf16(g), 0.0, gs, per_row=per_row, rstd_out=rstd)
    assert api.device_status() == 0
    _check(q, rstd, x, g, 0.0, per_row)


def test_special_values():
    """-0, subnormals, huge values, all-zero rows and a constant row."""
    M, K = 12, 1536
    x, g = _case(M, K, seed=90)
    x[0] = 0                      # all zero: ms 0, rstd = 1/sqrt(eps)
    x[1] = 0x8000                 # all -0
    x[2, ::3] = 0x0001            # subnormals
    x[3] = wl.f32_to_bf16_bits(np.full(K, 3.0, np.float32))
    x[4, :8] = 0x7F7F             # largest finite bf16: ms beyond fp32 -> rstd 0
    x[5, :4] = 0x5F80             # 2^64: squares beyond the fp32 range
    x[6] = wl.f32_to_bf16_bits(np.full(K, 1e-30, np.float32))
    for per_row in (False, True):
        rstd = torch.empty(M, dtype=torch.float32, device=DEV)
        gs = None if per_row else torch.tensor([1.0], dtype=torch.float32, device=DEV)
        q = api.nvfp4_rmsnorm_quantize(up_bf16(x), up_bf16(g), 1e-6, gs, per_row=per_row, rstd_out=rstd)
        assert api.device_status() == 0
        _check(q, rstd, x, g, 1e-6, per_row, np.float32(1.0))


def test_norm_stats_exact_path_equals_fast_path():
    """bsp_debug_norm_stats: the fp64 decision (with its exact fallback) and the
    exact integer sums alone give the same ms on every row, and 1/sqrt of it
    is the oracle's rstd."""
    x, _ = _case(600, 1536, seed=91)
    xb = np.concatenate([x, _midpoint_rows(1536, 30, seed=5)])
    xt = up_bf16(xb)
    (fast,), _ = api.norm_stats(xt, "rms")
    (exact,), p_exact = api.norm_stats(xt, "rms", exact_only=True)
    assert int(down(p_exact).min()) == 1
    assert torch.equal(fast, exact)
    r_ref = oracle.rmsnorm_rstd(xb, 0.0)
    r_gpu = np.array([oracle._rsqrt_rn32(np.float32(v)) for v in down(exact)], np.float32)
    assert np.array_equal(r_gpu.view(np.uint32), r_ref.view(np.uint32))


def test_equals_norm_then_quantize():
    """Same bytes as writing y = RMSNorm(x) in bf16 and quantizing it."""
    M, K = 300, 1536
    x, g = _case(M, K, seed=61)
    gs = torch.ones(1, dtype=torch.float32, device=DEV)
    fused = api.nvfp4_rmsnorm_quantize(up_bf16(x), up_bf16(g), 1e-6, gs)
    y = oracle.rmsnorm_bf16(x, g, oracle.rmsnorm_rstd(x, 1e-6))
    plain = api.nvfp4_quantize(up_bf16(y), gs)
    assert torch.equal(fused.codes, plain.codes) and torch.equal(fused.sf, plain.sf)


def test_norm_quantized_linear():
    M, N, K = 256, 768, 1536
    x, g = _case(M, K, seed=62)
    W = wl.f32_to_bf16_bits((np.random.default_rng(63).standard_normal((N, K)) * 0.02).astype(np.float32))
    layer = api.NVFP4Linear(up_bf16(W))
    xq = api.nvfp4_rmsnorm_quantize(up_bf16(x), up_bf16(g), 1e-6, layer.gs_x)
    D = layer(up_bf16(x), pre_quantized=xq)
    assert api.device_status() == 0
    ca, sa, _, _, _ = oracle.rmsnorm_quantize(x, g, 1e-6, np.float32(1.0))
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
    gk = g[:K].copy()
    q = api.nvfp4_rmsnorm_quantize(xs, up_bf16(gk), 1e-6, None, per_row=True, rstd_out=rstd)
    assert api.device_status() == 0
    _check(q, rstd, np.ascontiguousarray(x[:, :K]), gk, 1e-6, True)


@pytest.mark.parametrize("config", ["wan13", "wan14_in"])
def test_full_size_sampled_bands(config):
    """The full-size activation in the benchmark's launch configuration; the
    oracle checks sampled 128-row bands, the ragged last one included."""
    lin = getattr(wl, config)()
    from bench import norm_gamma
    g = norm_gamma(lin)
    M, K = lin.M, lin.K
    rstd = torch.empty(M, dtype=torch.float32, device=DEV)
    gs = torch.ones(1, dtype=torch.float32, device=DEV)
    q = api.nvfp4_rmsnorm_quantize(up_bf16(lin.A), up_bf16(g), 1e-6, gs, rstd_out=rstd)
    assert api.device_status() == 0
    for b in sample_bands(M, 3, seed=7):
        r0, r1 = b * 128, min(M, b * 128 + 128)
        codes, sf, r_ref, _, _ = oracle.rmsnorm_quantize(np.ascontiguousarray(lin.A[r0:r1]), g, 1e-6,
                                                         np.float32(1.0))
        assert np.array_equal(down(rstd[r0:r1]).view(np.uint32), r_ref.view(np.uint32)), b
        assert np.array_equal(down(q.codes[r0:r1]), codes), b
        assert np.array_equal(down(q.sf[b * 128 * (K // 16):(b + 1) * 128 * (K // 16)]), sf), b
