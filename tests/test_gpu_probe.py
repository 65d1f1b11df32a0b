"""The hardware conversions the quantize kernels use, against the oracle's
encoders, over every bf16 pattern, every rounding midpoint and its fp32
neighbours, signed zeros and subnormals; and the bounded-wait error path."""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_05_b200 import _native as nat
from tests._golden import e2m1_points
from tests._gpu import DEV, down, up

pytestmark = pytest.mark.gpu


def _probe_values():
    bits = np.arange(65536, dtype=np.uint32) << 16
    v = bits.view(np.float32)
    v = v[~np.isnan(v)]
    mids = []
    for grid in ([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0],
                 sorted({abs(oracle.e4m3_value(b)) for b in range(0x7F)})):
        g = np.array(grid, np.float64)
        m = ((g[1:] + g[:-1]) / 2).astype(np.float32)
        mids += [m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(1e9))]
    m = np.concatenate(mids)
    rng = np.random.default_rng(0)
    rnd = (rng.standard_normal(200000) * np.exp2(rng.integers(-30, 12, 200000))).astype(np.float32)
    tiny = np.array([1e-40, 1e-45, 1e-38, 2.0 ** -126, 2.0 ** -149], np.float32)
    specials = np.array([0.0, 448.0, 449.0, 464.0, 1e30, np.inf, 6.0, 6.5, 7.0, 1e9], np.float32)
    allv = np.concatenate([v, m, -m, rnd, tiny, -tiny, specials, -specials])
    return allv


def _run(fn, v):
    src = up(v.astype(np.float32))
    out = torch.empty(v.size, dtype=torch.uint8, device=DEV)
    nat.check(fn(src.data_ptr(), v.size, out.data_ptr(), torch.cuda.current_stream().cuda_stream), "probe")
    return down(out)


def test_hardware_e2m1_matches_oracle():
    v = _probe_values()
    got = _run(nat.lib().bsp_debug_encode_e2m1, v)
    want = oracle.e2m1_encode(v).astype(np.int16)
    bad = np.nonzero(got.astype(np.int16) != want)[0]
    assert bad.size == 0, [(float(v[i]), int(got[i]), int(want[i])) for i in bad[:12]]


def test_hardware_e2m1_golden_points():
    pts = e2m1_points()
    v = np.array([p[0] for p in pts], np.float32)
    got = _run(nat.lib().bsp_debug_encode_e2m1, v)
    assert [int(g) for g in got] == [p[1] for p in pts]


def test_hardware_e4m3_matches_oracle():
    v = _probe_values()
    got = _run(nat.lib().bsp_debug_encode_e4m3, v)
    want = oracle.e4m3_encode(v)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(v[i]), hex(int(got[i])), hex(int(want[i]))) for i in bad[:12]]


def test_bounded_wait_reports_timeout_and_context_survives():
    from block_scaled_precision_05_b200 import api
    assert api.device_status() == nat.BSP_OK
    nat.check(nat.lib().bsp_debug_wait_timeout(2_000_000, torch.cuda.current_stream().cuda_stream), "wait")
    assert api.device_status() == nat.BSP_ERR_TIMEOUT
    assert api.device_status() == nat.BSP_OK  # cleared
    x = torch.ones(4, device=DEV)
    assert float((x * 2).sum()) == 8.0  # the context still works
