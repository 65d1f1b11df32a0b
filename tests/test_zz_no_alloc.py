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


def _static(w, out):
    codes, sf, amax, gs, inv = out
    N, K = w.shape
    nat.check(nat.lib().nvfp4_quantize_weight_static(
        w.data_ptr(), nat.BSP_IN_BF16, N, K, w.stride(0), api.FP8_FP4_MAX, amax.data_ptr(), gs.data_ptr(),
        inv.data_ptr(), codes.data_ptr(), sf.data_ptr(), torch.cuda.current_stream().cuda_stream),
        "nvfp4_quantize_weight_static")


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
