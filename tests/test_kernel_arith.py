"""Arithmetic identities the CUDA quantizer relies on, proved exhaustively on
the CPU with exact rationals.

The group scale of NVFP4 (nvfp4_config.py, _nvfp4_quantize: the group amax
over 6, times the global scale) needs fl32(amax / 6).  The kernels compute it
as q = fl32(amax * fl32(1/6)) corrected once by the fma residual,
fl32(fma(fl32(fma(-q, 6, amax)), fl32(1/6), q)), with +inf passed through
(the amax of a group that holds an infinity); amax is always a bf16 or fp16
magnitude, so checking every such value proves the two equal."""
from fractions import Fraction

import numpy as np

import oracle


def _rn(fr: Fraction) -> np.float32:
    if fr < 0:
        return -_rn(-fr)
    return oracle._rn_f32_ratio(fr.numerator, fr.denominator)


def _f(x) -> Fraction:
    return Fraction(float(x))


def test_div6_by_corrected_product_is_correctly_rounded():
    sixth = np.float32(float.fromhex("0x1.555556p-3"))
    assert sixth == _rn(Fraction(1, 6))
    values = [np.uint32(b << 16).view(np.float32) for b in range(0, 0x7F80)]          # bf16, +0 and finite
    values += [np.float32(np.uint16(h).view(np.float16)) for h in range(0, 0x7C00)]  # fp16, +0 and finite
    single_product_misses = 0
    for x in values:
        want = _rn(_f(x) / 6)
        q = _rn(_f(x) * _f(sixth))
        r = _rn(-_f(q) * 6 + _f(x))            # fma(-q, 6, x): one rounding
        got = _rn(_f(r) * _f(sixth) + _f(q))   # fma(r, 1/6, q): one rounding
        assert got == want, x
        single_product_misses += q != want
    assert single_product_misses > 0  # the correction is needed
    # (+inf is passed through by the kernels: the residual would be inf - inf;
    # the GPU tests with infinite elements cover it)
