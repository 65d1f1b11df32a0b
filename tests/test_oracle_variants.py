"""Oracle pins for the global-scale variants: the 4over6 numerator
(sgl-project sglang nvfp4_online.py, _quantize_weight_nvfp4: e4m3_max = 256,
fp8_fp4_max = e4m3_max * 6) and one scale shared by a gated w1/w3 pair
(the same file, process_loaded_weight: the pair is concatenated along rows and
quantized with one amax-derived scale)."""
import numpy as np
import pytest

import oracle
from block_scaled_precision_05_b200 import workloads as wl


def _weights(rows, K, seed, std=0.02):
    rng = np.random.default_rng(seed)
    return wl.f32_to_bf16_bits((rng.standard_normal((rows, K)) * std).astype(np.float32))


def _e4m3_value(b):
    """Value of a non-negative e4m3 byte from its fields (exponent bias 7)."""
    b = np.asarray(b, dtype=np.int64)
    e, m = b >> 3, b & 7
    return np.where(e == 0, m / 8.0 * 2.0 ** -6, (1 + m / 8.0) * 2.0 ** (e - 7))


@pytest.mark.parametrize("amax,fmax,gs", [(6.0, 1536.0, 256.0), (6.0, 2688.0, 448.0), (3.0, 1536.0, 512.0),
                                          (1536.0, 1536.0, 1.0), (0.75, 1536.0, 2048.0), (0.0, 1536.0, 1.0)])
def test_global_scale_exact_cases(amax, fmax, gs):
    assert oracle.nvfp4_global_scale(amax, fmax) == np.float32(gs)


@pytest.mark.parametrize("fmax,top", [(1536.0, 256.0), (2688.0, 448.0)])
def test_group_scales_stop_at_e4m3_max(fmax, top):
    """With gs = e4m3_max*6/amax, the group holding the amax gets scale
    fl32(amax/6)*gs ~ e4m3_max and every other group less: the largest scale
    byte decodes to exactly e4m3_max (256 under 4over6, 448 otherwise)."""
    w = _weights(256, 512, seed=21)
    gs = oracle.nvfp4_global_scale(oracle.amax_bf16(w), fmax)
    _, sf = oracle.nvfp4_quantize(w, gs)
    vals = _e4m3_value(sf)
    assert vals.max() == top
    assert (vals <= top).all()


def test_shared_scale_pair_equals_split_of_concatenation():
    """Quantizing [w1; w3] with its amax equals quantizing w1 and w3 each with
    that shared scale: codes split by rows, scale tiles by 128-row bands."""
    w1, w3 = _weights(256, 320, seed=22), _weights(384, 320, seed=23, std=0.05)
    cat = np.concatenate([w1, w3], axis=0)
    gs = oracle.nvfp4_global_scale(oracle.amax_bf16(cat))
    assert gs == oracle.nvfp4_global_scale(max(oracle.amax_bf16(w1), oracle.amax_bf16(w3)))
    c_cat, s_cat = oracle.nvfp4_quantize(cat, gs)
    c1, s1 = oracle.nvfp4_quantize(w1, gs)
    c3, s3 = oracle.nvfp4_quantize(w3, gs)
    assert np.array_equal(c_cat, np.concatenate([c1, c3]))
    assert np.array_equal(s_cat, np.concatenate([s1, s3]))
