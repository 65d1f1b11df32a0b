"""Fused LayerNorm + NVFP4 quantize on the GPU against the oracle alone (the
producer of the pre-quantized activation of hao-ai-lab-FastVideo
nvfp4_config.py, NVFP4QuantizeMethod.apply, with the norm of the Wan-2.1
blocks).  Mean and variance are the exact values rounded once to fp32, so the
mean, rstd, y, the group scales and codes and the per-token scales all equal
the oracle's bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_05_b200 import api
from block_scaled_precision_05_b200 import workloads as wl
from tests._gpu import DEV, assert_gemm_close, down, sample_bands, up_bf16

pytestmark = pytest.mark.gpu


def _case(M, K, seed, shift=0.3):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((M, K)) + shift).astype(np.float32)
    x[rng.random((M, K)) < 0.001] *= 50
    g = (1.0 + 0.2 * rng.standard_normal(K)).astype(np.float32)
    b = (0.1 * rng.standard_normal(K)).astype(np.float32)
    return wl.f32_to_bf16_bits(x), wl.f32_to_bf16_bits(g), wl.f32_to_bf16_bits(b)


def _run(x, g, b, eps, per_row, gs=0.75):
    M = x.shape[0]
    mean = torch.empty(M, dtype=torch.float32, device=DEV)
    rstd = torch.empty(M, dtype=torch.float32, device=DEV)
    gst = None if per_row else torch.tensor([gs], dtype=torch.float32, device=DEV)
    q = api.nvfp4_layernorm_quantize(up_bf16(x), None if g is None else up_bf16(g), None if b is None else up_bf16(b),
                                     eps, gst, per_row=per_row, mean_out=mean, rstd_out=rstd)
    assert api.device_status() == 0
    return q, mean, rstd


def _check(q, mean, rstd, x, g, b, eps, per_row, gs=0.75):
    codes, sf, m_ref, r_ref, g_rows, inv_rows = oracle.layernorm_quantize(x, g, b, eps, np.float32(gs),
                                                                          per_row=per_row)
    assert np.array_equal(down(mean).view(np.uint32), m_ref.view(np.uint32))
    assert np.array_equal(down(rstd).view(np.uint32), r_ref.view(np.uint32))
    assert np.array_equal(down(q.codes), codes)
    assert np.array_equal(down(q.sf), sf)
    if per_row:
        assert np.array_equal(down(q.row_gs).view(np.uint32), g_rows.view(np.uint32))
        assert np.array_equal(down(q.row_inv_gs).view(np.uint32), inv_rows.view(np.uint32))


# K = 1536 and 2048 take the register-resident kernel, the others the
# multi-pass kernel
SHAPES = [(1, 16), (7, 48), (130, 1536), (300, 5120), (64, 13824), (129, 80), (257, 1024), (256, 2048),
          (1500, 1536), (129, 2048)]


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("per_row", [False, True])
def test_layernorm_quantize(M, K, per_row):
    x, g, b = _case(M, K, seed=M + 5 * K)
    q, mean, rstd = _run(x, g, b, 1e-6, per_row)
    _check(q, mean, rstd, x, g, b, 1e-6, per_row)


@pytest.mark.parametrize("affine", ["none", "gamma", "beta"])
@pytest.mark.parametrize("K", [1536, 640])
def test_optional_gamma_beta(affine, K):
    x, g, b = _case(200, K, seed=K + 11)
    g = g if affine == "gamma" else None
    b = b if affine == "beta" else None
    for per_row in (False, True):
        q, mean, rstd = _run(x, g, b, 1e-5, per_row)
        _check(q, mean, rstd, x, g, b, 1e-5, per_row)


def _tie_rows(K, n, seed):
    """Rows whose mean (K/2 elements 2, K/16 elements 2^-20: mean 1 + 2^-24) or
    whose variance (mean 0; K/8 each of +-2, K/32 each of +-2^-10: variance
    1 + 2^-24) lies exactly halfway between two fp32 values, scaled by powers
    of two and shuffled, and variants just off the tie.  The fp64 bound cannot
    decide them (nor any row whose mean is 0), so the exact sums do."""
    rng = np.random.default_rng(seed)
    rows = []
    for i in range(n):
        r = np.zeros(K, np.float32)
        if i % 2 == 0:
            r[: K // 2] = 2.0
            r[K // 2: K // 2 + K // 16] = 2.0 ** -20
            if i % 4 == 2:
                r = -r
        else:
            q8, q32 = K // 8, K // 32
            r[:q8], r[q8:2 * q8] = 2.0, -2.0
            r[2 * q8:2 * q8 + q32], r[2 * q8 + q32:2 * q8 + 2 * q32] = 2.0 ** -10, -(2.0 ** -10)
        if i % 3 == 1:
            r[-1] = 2.0 ** -50  # just off the tie
        r *= np.float32(2.0 ** rng.integers(-12, 12))
        rows.append(rng.permutation(r))
    return wl.f32_to_bf16_bits(np.stack(rows))


@pytest.mark.parametrize("K", [64, 1536, 2048, 5120])
@pytest.mark.parametrize("per_row", [False, True])
def test_rows_at_rounding_ties_take_the_exact_path(K, per_row):
    rand, g, b = _case(40, K, seed=K + 17)
    x = np.concatenate([_tie_rows(K, 24, seed=K), rand])
    _, path = api.norm_stats(up_bf16(x), "layer")
    assert int((down(path)[:24] != 0).sum()) >= 8  # the ties are not settled by the fp64 bounds
    q, mean, rstd = _run(x, g, b, 0.0, per_row)
    _check(q, mean, rstd, x, g, b, 0.0, per_row)


def test_special_values():
    """-0, subnormals, huge values, zero and constant rows, a mean far from 0."""
    M, K = 12, 1536
    x, g, b = _case(M, K, seed=92)
    x[0] = 0
    x[1] = 0x8000
    x[2, ::3] = 0x0001
    x[3] = wl.f32_to_bf16_bits(np.full(K, -3.0, np.float32))
    x[4, :8] = 0x7F7F  # variance beyond the fp32 range: rstd 0
    x[5, :4] = 0x5F80
    x[6] = wl.f32_to_bf16_bits(np.full(K, 1e-30, np.float32))
    x[7] = wl.f32_to_bf16_bits((np.random.default_rng(3).standard_normal(K) * 1e-3 + 1000.0).astype(np.float32))
    for per_row in (False, True):
        q, mean, rstd = _run(x, g, b, 1e-6, per_row, gs=1.0)
        _check(q, mean, rstd, x, g, b, 1e-6, per_row, gs=1.0)


def test_norm_stats_exact_path_equals_fast_path():
    x, _, _ = _case(600, 1536, seed=93)
    xb = np.concatenate([x, _tie_rows(1536, 30, seed=6)])
    xt = up_bf16(xb)
    (m_fast, v_fast), _ = api.norm_stats(xt, "layer")
    (m_ex, v_ex), p_ex = api.norm_stats(xt, "layer", exact_only=True)
    assert (down(p_ex) == 1).all()
    assert torch.equal(m_fast, m_ex) and torch.equal(v_fast, v_ex)
    m_ref, v_ref = oracle.layernorm_moments(xb)
    assert np.array_equal(down(m_ex).view(np.uint32), m_ref.view(np.uint32))
    assert np.array_equal(down(v_ex).view(np.uint32), v_ref.view(np.uint32))


def test_equals_norm_then_quantize():
    M, K = 300, 1536
    x, g, b = _case(M, K, seed=63)
    gs = torch.ones(1, dtype=torch.float32, device=DEV)
    fused = api.nvfp4_layernorm_quantize(up_bf16(x), up_bf16(g), up_bf16(b), 1e-6, gs)
    mean, rstd = oracle.layernorm_stats(x, 1e-6)
    y = oracle.layernorm_bf16(x, g, b, mean, rstd)
    plain = api.nvfp4_quantize(up_bf16(y), gs)
    assert torch.equal(fused.codes, plain.codes) and torch.equal(fused.sf, plain.sf)


def test_norm_quantized_linear():
    M, N, K = 256, 768, 5120
    x, g, b = _case(M, K, seed=64)
    W = wl.f32_to_bf16_bits((np.random.default_rng(65).standard_normal((N, K)) * 0.02).astype(np.float32))
    layer = api.NVFP4Linear(up_bf16(W), per_token=True)
    xq = layer.layernorm_quantize_input(up_bf16(x), up_bf16(g), up_bf16(b), 1e-6)
    D = layer(up_bf16(x), pre_quantized=xq)
    assert api.device_status() == 0
    ca, sa, _, _, _, inv = oracle.layernorm_quantize(x, g, b, 1e-6, per_row=True)
    gso = oracle.nvfp4_global_scale(oracle.amax_bf16(W))
    cb, sb = oracle.nvfp4_quantize(W, gso)
    ref, bound = oracle.linear_reference(oracle.nvfp4_dequantize(ca, sa, K), oracle.nvfp4_dequantize(cb, sb, K),
                                         alpha=np.float32(1) / gso, row_scale=inv, bias=None)
    assert_gemm_close(D, ref, bound, "layernorm-quantized linear")


@pytest.mark.parametrize("K", [1536, 1024])
def test_strided_rows(K):
    M = 200
    x, g, b = _case(M, K + 64, seed=K + 9)
    xs = up_bf16(x)[:, :K]
    mean = torch.empty(M, dtype=torch.float32, device=DEV)
    rstd = torch.empty(M, dtype=torch.float32, device=DEV)
    gk, bk = g[:K].copy(), b[:K].copy()
    q = api.nvfp4_layernorm_quantize(xs, up_bf16(gk), up_bf16(bk), 1e-6, None, per_row=True, mean_out=mean,
                                     rstd_out=rstd)
    assert api.device_status() == 0
    _check(q, mean, rstd, np.ascontiguousarray(x[:, :K]), gk, bk, 1e-6, True)


@pytest.mark.parametrize("config", ["wan13", "wan14_in"])
def test_full_size_sampled_bands(config):
    """The full-size activation in the benchmark's launch configuration; the
    oracle checks sampled 128-row bands, the ragged last one included."""
    lin = getattr(wl, config)()
    from bench import norm_beta, norm_gamma
    g, b = norm_gamma(lin), norm_beta(lin)
    M, K = lin.M, lin.K
    mean = torch.empty(M, dtype=torch.float32, device=DEV)
    rstd = torch.empty(M, dtype=torch.float32, device=DEV)
    gs = torch.ones(1, dtype=torch.float32, device=DEV)
    q = api.nvfp4_layernorm_quantize(up_bf16(lin.A), up_bf16(g), up_bf16(b), 1e-6, gs, mean_out=mean, rstd_out=rstd)
    assert api.device_status() == 0
    for bd in sample_bands(M, 3, seed=8):
        r0, r1 = bd * 128, min(M, bd * 128 + 128)
        codes, sf, m_ref, r_ref, _, _ = oracle.layernorm_quantize(np.ascontiguousarray(lin.A[r0:r1]), g, b, 1e-6,
                                                                  np.float32(1.0))
        assert np.array_equal(down(mean[r0:r1]).view(np.uint32), m_ref.view(np.uint32)), bd
        assert np.array_equal(down(rstd[r0:r1]).view(np.uint32), r_ref.view(np.uint32)), bd
        assert np.array_equal(down(q.codes[r0:r1]), codes), bd
        assert np.array_equal(down(q.sf[bd * 128 * (K // 16):(bd + 1) * 128 * (K // 16)]), sf), bd
