"""Pins of the oracle's 8x4 scale layout (hao-ai-lab-FastVideo
nvfp4_config.py: SfLayout.layout_8x4 with rows padded to 8, mm_fp4's
use_8x4_sf_layout).  The pages do not give the byte order inside a tile; the
reading is a row-major 8x4 tile of 32 bytes, tiles ordered by row tile then
column tile."""
import numpy as np
import pytest

import oracle
from block_scaled_precision_05_b200 import workloads as wl


@pytest.mark.parametrize("rows,cols", [(1, 4), (8, 4), (9, 6), (64, 96), (130, 13)])
def test_map_is_a_bijection(rows, cols):
    cols_p = -(-cols // 4) * 4
    rows_p = -(-rows // 8) * 8
    offs = [oracle.sf_offset(r, c, cols_p, "8x4") for r in range(rows_p) for c in range(cols_p)]
    assert sorted(offs) == list(range(oracle.sf_bytes(rows, cols, "8x4")))


@pytest.mark.parametrize("rows,cols", [(8, 4), (24, 12), (64, 96)])
def test_map_equals_blocked_reshape(rows, cols):
    """Logical [rows, cols] -> [rows/8, cols/4, 8, 4] blocks, flattened."""
    logical = np.arange(rows * cols).reshape(rows, cols)
    blocked = logical.reshape(rows // 8, 8, cols // 4, 4).transpose(0, 2, 1, 3).reshape(-1)
    buf = np.empty(rows * cols, np.int64)
    for r in range(rows):
        for c in range(cols):
            buf[oracle.sf_offset(r, c, cols, "8x4")] = logical[r, c]
    assert np.array_equal(buf, blocked)


def _logical(sf, rows, cols, layout):
    cols_p = -(-cols // 4) * 4
    return np.array([[sf[oracle.sf_offset(r, c, cols_p, layout)] for c in range(cols)] for r in range(rows)])


@pytest.mark.parametrize("M,K", [(1, 64), (13, 80), (64, 512)])
def test_layouts_hold_the_same_scales(M, K):
    x = wl.f32_to_bf16_bits(np.random.default_rng(M + K).standard_normal((M, K)).astype(np.float32))
    c1, s1 = oracle.nvfp4_quantize(x, np.float32(1.0))
    c8, s8 = oracle.nvfp4_quantize(x, np.float32(1.0), layout="8x4")
    assert np.array_equal(c1, c8)
    assert np.array_equal(_logical(s1, M, K // 16, "128x4"), _logical(s8, M, K // 16, "8x4"))
    # every byte outside the logical scales is padding, and zero
    assert s8.size == oracle.sf_bytes(M, K // 16, "8x4")
    assert int(s8.sum()) == int(_logical(s8, M, K // 16, "8x4").sum())
    assert np.array_equal(oracle.nvfp4_dequantize(c1, s1, K), oracle.nvfp4_dequantize(c8, s8, K, layout="8x4"))
