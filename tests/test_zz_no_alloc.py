"""nvfp4_quantize_weight_static -- the weight conversion whose scratch is a
static device array inside the library (no workspace argument, no
allocation) -- against nvfp4_quantize_weight with a caller workspace: two
calls in a row, on different weights, give the same codes, scales and global
scales.  Collected last, and independent of what ran before it."""
import pytest
import torch

from block_scaled_precision_05_b200 import _native as nat
from block_scaled_precision_05_b200 import api

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def _outputs(N, K):
    return (torch.empty((N, K // 2), dtype=torch.uint8, device=DEV),
            torch.empty(api.nvfp4_sf_bytes(N, K), dtype=torch.uint8, device=DEV),
            *(torch.empty(1, dtype=torch.float32, device=DEV) for _ in range(3)))


def _static(w, out, fmax=api.FP8_FP4_MAX):
    codes, sf, amax, gs, inv = out
    N, K = w.shape
    w_dtype = nat.BSP_IN_F16 if w.dtype == torch.float16 else nat.BSP_IN_BF16
    nat.check(nat.lib().nvfp4_quantize_weight_static(
        w.data_ptr(), w_dtype, N, K, w.stride(0), fmax, amax.data_ptr(), gs.data_ptr(),
        inv.data_ptr(), codes.data_ptr(), sf.data_ptr(), torch.cuda.current_stream().cuda_stream),
        "nvfp4_quantize_weight_static")


def _same(out, ref):
    codes, sf, amax, gs, inv = out
    q, gs_r, inv_r, amax_r = ref
    assert torch.equal(codes, q.codes) and torch.equal(sf, q.sf)
    assert torch.equal(gs, gs_r) and torch.equal(inv, inv_r) and torch.equal(amax, amax_r)


def test_static_scratch_matches_workspace_entry():
    g = torch.Generator(device=DEV)
    g.manual_seed(2024)
    weights = [(torch.randn((5120, 5120), generator=g, device=DEV) * 0.02).to(torch.bfloat16),
               (torch.randn((1000, 1536), generator=g, device=DEV) * 3.0).to(torch.bfloat16)]
    outs = [_outputs(*w.shape) for w in weights]
    for w, out in zip(weights, outs):  # two calls in a row, no synchronisation between them
        _static(w, out)
    refs = [api.nvfp4_quantize_weight(w) for w in weights]
    torch.cuda.synchronize()
    assert api.device_status() == 0
    for (codes, sf, amax, gs, inv), (q, gs_r, inv_r, amax_r) in zip(outs, refs):
        assert torch.equal(codes, q.codes) and torch.equal(sf, q.sf)
        assert torch.equal(gs, gs_r) and torch.equal(inv, inv_r) and torch.equal(amax, amax_r)


def test_static_scratch_fp16_strided_ragged_and_after_batch():
    """fp16 weights, a row stride wider than K, N not a multiple of 128, 4over6,
    and a call right after nvfp4_quantize_weights has used the caller-workspace
    path: each matches nvfp4_quantize_weight on the same weight."""
    g = torch.Generator(device=DEV)
    g.manual_seed(2025)
    big = (torch.randn((333, 1600), generator=g, device=DEV) * 0.5).to(torch.float16)
    cases = [(big[:, :1536], api.FP8_FP4_MAX),
             ((torch.randn((130, 640), generator=g, device=DEV) * 3.0).to(torch.bfloat16), api.FP8_FP4_MAX_4OVER6)]
    api.nvfp4_quantize_weights([(torch.randn((256, 1024), generator=g, device=DEV)).to(torch.bfloat16)])
    for w, fmax in cases:
        out = _outputs(*w.shape)
        _static(w, out, fmax)
        ref = api.nvfp4_quantize_weight(w, fmax)
        torch.cuda.synchronize()
        assert api.device_status() == 0
        _same(out, ref)


def test_static_scratch_rejects_bad_arguments_before_any_launch():
    L = nat.lib()
    st = torch.cuda.current_stream().cuda_stream
    w = torch.zeros((128, 64), dtype=torch.bfloat16, device=DEV)
    codes, sf, amax, gs, inv = _outputs(128, 64)
    p = [t.data_ptr() for t in (amax, gs, inv, codes, sf)]
    bad = [
        (w.data_ptr(), nat.BSP_IN_BF16, 128, 48, 64, api.FP8_FP4_MAX),   # K % 64 != 0
        (w.data_ptr(), nat.BSP_IN_BF16, 128, 64, 32, api.FP8_FP4_MAX),   # ld_w < K
        (w.data_ptr(), nat.BSP_IN_BF16, -1, 64, 64, api.FP8_FP4_MAX),    # N < 0
        (w.data_ptr(), 7, 128, 64, 64, api.FP8_FP4_MAX),                  # unknown input format
        (w.data_ptr(), nat.BSP_IN_BF16, 128, 64, 64, -1.0),               # fp8_fp4_max <= 0
        (None, nat.BSP_IN_BF16, 128, 64, 64, api.FP8_FP4_MAX),           # no weight
    ]
    for args in bad:
        assert L.nvfp4_quantize_weight_static(*args, *p, st) == nat.BSP_ERR_INVALID_ARG, args
    torch.cuda.synchronize()
    assert api.device_status() == 0
