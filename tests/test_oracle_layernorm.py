"""Pins of the oracle's LayerNorm reading (the norm in front of the quantizer
in the Wan-2.1 blocks; hao-ai-lab-FastVideo nvfp4_config.py names fused
norm+quant producers of the pre-quantized activation but not the norm):
  mean = mean(x) and var = mean((x - mean)^2), each exact and rounded once to
  fp32; rstd = RN32(1/sqrt(RN32(var+eps)));
  y = bf16(RN32(RN32(RN32(RN32(x - mean)*rstd)*gamma) + beta)).
The exact values are recomputed here with Fractions in the two-pass form of
the definition (the oracle uses the one-pass integer identity), and the
oracle's fp32 results must be the correctly rounded ones."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_05_b200 import workloads as wl


def _bits(a):
    return wl.f32_to_bf16_bits(np.asarray(a, np.float32))


def _is_rn32(r: np.float32, q: Fraction) -> bool:
    """r is the fp32 nearest to q, ties to even (finite r)."""
    r = np.float32(r)
    d = abs(Fraction(float(r)) - q)
    for nb in (np.nextafter(r, np.float32(-np.inf), dtype=np.float32),
               np.nextafter(r, np.float32(np.inf), dtype=np.float32)):
        dn = abs(Fraction(float(nb)) - q)
        if dn < d:
            return False
        if dn == d and (r.view(np.uint32) & 1):
            return False
    return True


def _exact_two_pass(row_bits):
    xs = [Fraction(float(v)) for v in oracle.bf16_bits_to_f64(row_bits)]
    mu = sum(xs) / len(xs)
    var = sum((v - mu) ** 2 for v in xs) / len(xs)
    return mu, var


@pytest.mark.parametrize("c", [2.0, -0.5, 1.0, 3.0, 0.0])
def test_constant_rows(c):
    x = _bits(np.full((1, 32), c))
    mean, var = oracle.layernorm_moments(x)
    assert mean[0] == np.float32(c) and var[0] == 0.0
    _, rstd = oracle.layernorm_stats(x, 0.25)
    assert rstd[0] == np.float32(2.0)  # 1/sqrt(0 + 0.25)
    beta = _bits(np.linspace(-1, 1, 32))
    y = oracle.layernorm_bf16(x, None, beta, mean, rstd)
    assert (y == beta).all()  # (x - mean) * rstd = 0, then + beta


@pytest.mark.parametrize("a,b,mean,var", [(3.0, 1.0, 2.0, 1.0), (1.5, -0.5, 0.5, 1.0), (-4.0, 4.0, 0.0, 16.0),
                                          (0.75, 0.25, 0.5, 0.0625)])
def test_two_valued_rows_closed_form(a, b, mean, var):
    x = _bits(np.array([[a, b] * 24]))
    m, v = oracle.layernorm_moments(x)
    assert m[0] == np.float32(mean) and v[0] == np.float32(var)
    _, rstd = oracle.layernorm_stats(x, 0.0)
    y = oracle.layernorm_bf16(x, None, None, m, rstd)
    assert (y[0, 0::2] == _bits([1.0 if a > b else -1.0])[0]).all()


def test_correct_rounding_against_two_pass_fractions():
    rng = np.random.default_rng(60)
    rows = [rng.standard_normal(64) * 3 + 0.7,
            rng.standard_normal(64) * 1e-3 + 5.0,            # mean far from 0
            rng.standard_normal(64) * 1e4,
            rng.standard_normal(64) * 1e-30,                 # tiny values
            np.where(rng.random(64) < 0.05, 300.0, rng.standard_normal(64))]
    x = _bits(np.stack(rows))
    x[3, :5] = 0x0003  # subnormals
    x[1, 7] = 0x8000   # -0
    mean, var = oracle.layernorm_moments(x)
    for r in range(x.shape[0]):
        mu, v = _exact_two_pass(x[r])
        assert _is_rn32(mean[r], mu), r
        assert _is_rn32(var[r], v), r


def test_midpoints_round_to_even():
    # mean exactly halfway between 1 and 1 + 2^-23: 32 x 2.0 and 4 x 2^-20 in 64 -> 1 + 2^-24
    row = np.zeros(64, np.float32)
    row[:32] = 2.0
    row[32:36] = 2.0 ** -20
    x = _bits(row[None])
    mean, _ = oracle.layernorm_moments(x)
    assert mean[0] == np.float32(1.0)
    row[40] = 2.0 ** -60  # just above the tie
    mean, _ = oracle.layernorm_moments(_bits(row[None]))
    assert mean[0] == np.nextafter(np.float32(1.0), np.float32(2.0))
    # var exactly at 1 + 2^-24 with mean 0: +-2 on 8 each, +-2^-10 on 2 each, in 64
    row = np.zeros(64, np.float32)
    row[:8], row[8:16] = 2.0, -2.0
    row[16:18], row[18:20] = 2.0 ** -10, -(2.0 ** -10)
    mean, var = oracle.layernorm_moments(_bits(row[None]))
    assert mean[0] == 0.0 and not np.signbit(mean[0])
    assert var[0] == np.float32(1.0)


def test_smallest_means_are_exact_subnormals():
    # bf16 values are multiples of 2^-133, so a nonzero mean is at least 2^-133 / K
    # (>= 2^-148 for K <= 2^15): never rounded to zero
    x = np.zeros((2, 16), np.uint16)
    x[0, 3] = 0x8001  # -2^-133
    x[1, 5] = 0x0003  # 3 * 2^-133
    mean, var = oracle.layernorm_moments(x)
    assert mean[0] == np.float32(-(2.0 ** -137)) and mean[1] == np.float32(3 * 2.0 ** -137)
    assert var[0] == 0.0  # 15 * 2^-274 / 256: far below the smallest subnormal


def test_absent_gamma_beta_are_identities():
    rng = np.random.default_rng(61)
    x = _bits(rng.standard_normal((8, 128)))
    x[0, :4] = 0x8000
    mean, rstd = oracle.layernorm_stats(x, 1e-6)
    ones = _bits(np.ones(128))
    negz = np.full(128, 0x8000, np.uint16)
    base = oracle.layernorm_bf16(x, None, None, mean, rstd)
    assert (oracle.layernorm_bf16(x, ones, None, mean, rstd) == base).all()
    assert (oracle.layernorm_bf16(x, ones, negz, mean, rstd) == base).all()


def test_matches_torch_layer_norm_within_one_bf16_ulp():
    rng = np.random.default_rng(62)
    x = _bits(rng.standard_normal((40, 512)) * 3 + 0.5)
    g = _bits(1 + 0.1 * rng.standard_normal(512))
    b = _bits(0.1 * rng.standard_normal(512))
    mean, rstd = oracle.layernorm_stats(x, 1e-6)
    y = oracle.layernorm_bf16(x, g, b, mean, rstd)
    xt = torch.from_numpy(oracle.bf16_bits_to_f64(x))
    ref = torch.nn.functional.layer_norm(xt, (512,), weight=torch.from_numpy(oracle.bf16_bits_to_f64(g)),
                                         bias=torch.from_numpy(oracle.bf16_bits_to_f64(b)), eps=1e-6).numpy()
    got = oracle.bf16_bits_to_f64(y)
    ulp = np.abs(oracle.bf16_bits_to_f64(oracle.bf16_round(ref) + 1) - oracle.bf16_bits_to_f64(oracle.bf16_round(ref)))
    assert (np.abs(got - ref) <= ulp).all()
    v64, m64 = torch.var_mean(xt, dim=1, unbiased=False)
    m_o, v_o = oracle.layernorm_moments(x)
    assert np.all(np.abs(m_o - m64.numpy()) <= np.spacing(np.abs(m_o)))
    assert np.all(np.abs(v_o - v64.numpy()) <= np.spacing(np.abs(v_o)))


def test_variance_beyond_fp32_rounds_to_inf_and_rstd_to_zero():
    # +-2^64 alternating: mean 0, var = 2^128 exactly, above the largest finite
    # fp32 and past the midpoint to it, so RN32 gives +inf; then rstd =
    # RN32(1/sqrt(inf)) = 0 and y = ((x - 0) * 0) * 1 + beta = beta
    x = _bits(np.array([[2.0 ** 64, -(2.0 ** 64)] * 16]))
    mean, var = oracle.layernorm_moments(x)
    assert mean[0] == 0.0 and np.isposinf(var[0])
    m, rstd = oracle.layernorm_stats(x, 1e-6)
    assert rstd[0] == 0.0
    beta = _bits(np.linspace(-1, 1, 32))
    assert (oracle.layernorm_bf16(x, None, beta, m, rstd) == beta).all()
    # +-255 * 2^56: var = 65025 * 2^112 = 16646400 * 2^104, exact in fp32 (below 2^24 * 2^104)
    x = _bits(np.array([[255 * 2.0 ** 56, -255 * 2.0 ** 56] * 16]))
    mean, var = oracle.layernorm_moments(x)
    assert mean[0] == 0.0 and var[0] == np.float32(16646400 * 2.0 ** 104)
