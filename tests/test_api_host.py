"""Host-side behaviour of the Python binding (no GPU needed): inputs are
coerced by the pages' dtype rule, and every entry point refuses CPU tensors
instead of computing anything on the host -- there is no CPU path."""
import pytest
import torch

from block_scaled_precision_05_b200 import api


def test_input_dtype_rule():
    b = torch.zeros(4, 16, dtype=torch.bfloat16)
    h = torch.zeros(4, 16, dtype=torch.float16)
    assert api.coerce_input(b) is b and api.coerce_input(h) is h
    assert api.coerce_input(torch.zeros(4, 16)).dtype == torch.bfloat16
    assert api.coerce_bf16(h).dtype == torch.bfloat16
    with pytest.raises(TypeError):
        api.coerce_input(torch.zeros(4, 16, dtype=torch.int32))


def test_cpu_tensors_are_refused():
    x = torch.zeros(32, 64, dtype=torch.bfloat16)
    gs = torch.ones(1)
    calls = [
        lambda: api.amax(x),
        lambda: api.nvfp4_quantize(x, gs),
        lambda: api.nvfp4_quantize(x, per_row=True),
        lambda: api.mxfp8_quantize(x),
        lambda: api.nvfp4_rmsnorm_quantize(x, torch.ones(64, dtype=torch.bfloat16), 1e-6, gs),
        lambda: api.nvfp4_quantize_weight(x),
        lambda: api.nvfp4_quantize_weights([x, x]),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA"):
            call()


def test_weight_batch_edge_cases():
    assert api.nvfp4_quantize_weights([]) == []
    with pytest.raises(ValueError):
        api.nvfp4_quantize_weights([torch.zeros(4, 48, dtype=torch.bfloat16)])
