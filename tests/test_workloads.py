"""The seeded synthetic inputs have the shapes and distributions of the five
workload configurations (the DiT-shaped layers, their outliers, the GELU
input of fc_out, the skinny sweep and the 40-block weight stack), and are
reproducible from their seeds."""
import math

import numpy as np

from block_scaled_precision_05_b200 import workloads as wl


def _f(bits):
    return wl.bf16_bits_to_f32(bits).astype(np.float64)


def test_shapes():
    assert (wl.tiny().A.shape, wl.tiny().W.shape) == ((128, 256), (256, 256))
    small = 256  # the activation row count is a parameter; the layer shapes are fixed
    assert wl.wan14_in(M=small).W.shape == (13824, 5120) and wl.wan14_in(M=small).A.shape == (small, 5120)
    assert wl.wan14_out(M=small).W.shape == (5120, 13824) and wl.wan14_out(M=small).A.shape == (small, 13824)
    assert wl.mxfp8(M=small).W.shape == (5120, 5120)
    for M in (1, 16, 128):
        lin = wl.skinny(M)
        assert lin.A.shape == (M, 5120) and lin.W.shape == (13824, 5120) and lin.per_token
    shapes = wl.dit_weight_shapes(40)
    assert len(shapes) == 240
    assert sum(N * K for (_, _, N, K) in shapes) == 40 * (4 * 5120 * 5120 + 2 * 13824 * 5120)


def test_wan13_distributions():
    lin = wl.wan13()
    assert lin.A.shape == (32760, 1536) and lin.W.shape == (1536, 1536) and lin.bias.shape == (1536,)
    A, W, b = _f(lin.A), _f(lin.W), _f(lin.bias)
    big = np.abs(A) > 8.0  # ~1e-15 for N(0, 1): these are the x50 outliers
    frac = big.mean()
    assert 0.0007 < frac < 0.0011, frac  # Bernoulli(0.001), about half of them above 8
    assert abs(A[~big].std() - 1.0) < 0.01
    assert abs(W.std() * math.sqrt(1536) - 1.0) < 0.01
    assert abs(b.std() / 0.01 - 1.0) < 0.1


def test_fc_out_input_is_gelu():
    A = _f(wl.wan14_out(M=512).A)
    assert A.min() > -0.18  # GELU_tanh is bounded below by about -0.17
    assert 0.2 < (A < 0).mean() < 0.6  # small negative lobe, positive tail


def test_seeded():
    assert np.array_equal(wl.wan13(M=64).A, wl.wan13(M=64).A)
    assert np.array_equal(wl.skinny(16).W, wl.skinny(128).W)  # one weight for the whole sweep
    assert not np.array_equal(wl.skinny(16).A, wl.skinny(16, seed=9).A)
