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


# --------------------------------------------------------------------------- fp16 input
# nvfp4_config.py (_coerce_fp4_input_dtype, NVFP4QuantizeMethod.apply) feeds
# fp16 activations to the quantizer as they are.

def test_f16_decoder_matches_numpy_on_every_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_value(int(b)) for b in bits])
    r = ref
    same = (got == r) | (np.isnan(got) & np.isnan(r))
    assert same.all()


def test_f16_amax_nan_and_inf():
    x = np.array([0x3C00, 0xBC00, 0x7E00, 0x4000], np.uint16)  # 1, -1, NaN, 2
    assert oracle.amax_f16(x) == 2.0
    assert oracle.amax_f16(np.array([0x3C00, 0xFC00], np.uint16)) == 65504.0  # -inf -> largest finite
    assert oracle.amax_f16(np.array([0x7E00, 0x8000], np.uint16)) == 0.0


def test_f16_and_bf16_agree_on_shared_values():
    """Values representable in both formats quantize identically."""
    rng = np.random.default_rng(41)
    vals = (rng.integers(-64, 65, size=(130, 96)) / 8.0).astype(np.float32)  # k/8: exact in both
    b16 = wl.f32_to_bf16_bits(vals)
    f16 = vals.astype(np.float16).view(np.uint16)
    for per_row in (False, True):
        if per_row:
            gs_b, _ = oracle.row_global_scales(b16)
            gs_f, _ = oracle.row_global_scales(f16, fmt="f16")
            assert np.array_equal(gs_b, gs_f)
        else:
            gs_b = gs_f = oracle.nvfp4_global_scale(oracle.amax_bf16(b16))
        cb, sb = oracle.nvfp4_quantize(b16, gs_b, per_row=per_row)
        cf, sf = oracle.nvfp4_quantize(f16, gs_f, per_row=per_row, fmt="f16")
        assert np.array_equal(cb, cf) and np.array_equal(sb, sf)


def test_f16_precision_is_used():
    """1.25 + 2^-10 is just above the e2m1 tie between 1 and 1.5: in fp16 it
    rounds up to 1.5 (code 3); rounded to bf16 first it is the tie itself,
    which goes to the even code 2 (1.0).  Group scale 1: the 6.0 sets amax."""
    f16 = np.zeros((1, 16), np.uint16)
    f16[0, 0] = np.float16(6.0).view(np.uint16)
    f16[0, 1] = np.float16(1.2509765625).view(np.uint16)
    codes, sf = oracle.nvfp4_quantize(f16, np.float32(1.0), fmt="f16")
    assert sf[0] == 0x38  # e4m3 1.0
    assert codes[0, 0] == (0x7 | (0x3 << 4))
    b16 = wl.f32_to_bf16_bits(np.array([[6.0, 1.2509765625] + [0.0] * 14], np.float32))
    codes_b, _ = oracle.nvfp4_quantize(b16, np.float32(1.0))
    assert codes_b[0, 0] == (0x7 | (0x2 << 4))
