"""Pins of the oracle's RMSNorm reading (the norm in front of the quantizer;
hao-ai-lab-FastVideo nvfp4_config.py names fused norm+quant producers of the
pre-quantized activation but not the norm):
  ms = mean(x^2) exactly, rounded once to fp32; rstd = RN32(1/sqrt(RN32(ms+eps)));
  y = bf16(RN32(RN32(x*rstd)*gamma))."""
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_05_b200 import workloads as wl


def _bits(a):
    return wl.f32_to_bf16_bits(np.asarray(a, np.float32))


@pytest.mark.parametrize("c,eps,rstd,y", [(2.0, 0.0, 0.5, 1.0), (-0.5, 0.0, 2.0, -1.0), (1.0, 3.0, 0.5, 0.5),
                                          (3.0, 0.0, np.float32(1.0) / np.float32(3.0), 1.0)])
def test_constant_rows(c, eps, rstd, y):
    x = _bits(np.full((1, 32), c))
    g = _bits(np.ones(32))
    r = oracle.rmsnorm_rstd(x, eps)
    assert r[0] == np.float32(rstd)
    out = oracle.rmsnorm_bf16(x, g, r)
    assert (out == _bits([y])[0]).all()


def test_gamma_scales_after_normalising():
    x = _bits(np.full((1, 16), 2.0))
    g = _bits(np.array([1.0, -2.0, 0.5, 0.0] * 4))
    out = oracle.rmsnorm_bf16(x, g, oracle.rmsnorm_rstd(x, 0.0))
    assert (out[0, :4] == _bits([1.0, -2.0, 0.5, 0.0])).all()


def test_ratio_rounding_exact_values_and_midpoints():
    rng = np.random.default_rng(50)
    vals = rng.standard_normal(300).astype(np.float32)
    vals = np.abs(vals[vals != 0])
    for v in vals:
        f = Fraction(float(v))
        assert oracle._rn_f32_ratio(f.numerator, f.denominator) == v
        b = np.nextafter(v, np.float32(np.inf), dtype=np.float32)
        mid = (Fraction(float(v)) + Fraction(float(b))) / 2
        even = v if (v.view(np.uint32) & 1) == 0 else b
        assert oracle._rn_f32_ratio(mid.numerator, mid.denominator) == even
        above = mid + Fraction(1, mid.denominator * 4)
        below = mid - Fraction(1, mid.denominator * 4)
        assert oracle._rn_f32_ratio(above.numerator, above.denominator) == b
        assert oracle._rn_f32_ratio(below.numerator, below.denominator) == v
    # subnormal result and zero
    tiny = Fraction(3, 2 ** 150)
    assert oracle._rn_f32_ratio(tiny.numerator, tiny.denominator) == np.float32(2.0 ** -149) * 2
    assert oracle._rn_f32_ratio(0, 7) == 0


def test_rsqrt_against_high_precision():
    getcontext().prec = 60
    rng = np.random.default_rng(51)
    ts = np.abs(rng.standard_normal(400).astype(np.float32)) * np.float32(10.0) ** rng.integers(-6, 6, 400)
    ts = ts[ts > 0].astype(np.float32)
    for t in list(ts) + [np.float32(4.0), np.float32(0.25), np.float32(1.0 / 16)]:
        got = oracle._rsqrt_rn32(np.float32(t))
        z = Decimal(1) / Decimal(float(t)).sqrt()
        a = np.float32(got)
        for nb in (np.nextafter(a, np.float32(0), dtype=np.float32),
                   np.nextafter(a, np.float32(np.inf), dtype=np.float32)):
            assert abs(Decimal(float(a)) - z) <= abs(Decimal(float(nb)) - z)


def test_matches_torch_rms_norm_within_one_bf16_ulp():
    rng = np.random.default_rng(52)
    x = _bits(rng.standard_normal((40, 512)) * 3)
    g = _bits(1 + 0.1 * rng.standard_normal(512))
    y = oracle.rmsnorm_bf16(x, g, oracle.rmsnorm_rstd(x, 1e-6))
    xt = torch.from_numpy(oracle.bf16_bits_to_f64(x))
    gt = torch.from_numpy(oracle.bf16_bits_to_f64(g))
    ref = torch.nn.functional.rms_norm(xt, (512,), weight=gt, eps=1e-6).numpy()
    got = oracle.bf16_bits_to_f64(y)
    ulp = np.abs(oracle.bf16_bits_to_f64(oracle.bf16_round(ref) + 1) - oracle.bf16_bits_to_f64(oracle.bf16_round(ref)))
    assert (np.abs(got - ref) <= ulp).all()


def test_rsqrt_at_zero_and_infinity_and_overflowing_mean():
    assert oracle._rsqrt_rn32(np.float32(np.inf)) == 0.0
    assert oracle._rsqrt_rn32(np.float32(0.0)) == np.float32(np.inf)
    # squares of the largest bf16 overflow the fp32 mean: ms = inf, rstd = +0, y = 0
    x = np.zeros((1, 32), np.uint16)
    x[0, :4] = 0x7F7F
    r = oracle.rmsnorm_rstd(x, 1e-6)
    assert r[0] == 0.0 and not np.signbit(r[0])
    y = oracle.rmsnorm_bf16(x, _bits(np.ones(32)), r)
    assert (y & 0x7FFF == 0).all()
