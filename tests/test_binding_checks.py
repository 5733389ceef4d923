"""The Python binding's own argument checks (they raise before any device work, so they
run without a GPU): shapes and dtypes of the newer calls, and CPU tensors refused."""
import pytest
import torch

from linear_attention_sequence_mshortconv_b200 import kda


def _scan_inputs(B=1, T=8, H=2, D=32, dtype=torch.float32):
    z = lambda *s: torch.zeros(*s, dtype=dtype)
    return z(B, T, H, D), z(B, T, H, D), z(B, T, H, D), z(B, T, H, D), z(B, T, H)


def test_backward_checks_shapes_and_devices():
    q, k, v, g, beta = _scan_inputs()
    with pytest.raises(ValueError):
        kda.backward(q, k, v, g, beta[:, :4], torch.zeros(1, 8, 2, 32))     # beta length
    with pytest.raises(ValueError):
        kda.backward(q, k, v, g, beta, torch.zeros(1, 8, 2, 16))            # do width
    with pytest.raises(TypeError):
        kda.backward(q, k, v, g.double(), beta, torch.zeros(1, 8, 2, 32))   # mixed dtypes
    with pytest.raises(TypeError):   # host tensors are refused (no CPU path)
        kda.backward(q, k, v, g, beta, torch.zeros(1, 8, 2, 32))


def test_sequence_parallel_calls_check_shapes():
    with pytest.raises(ValueError):
        kda.sp_prefix(torch.zeros(2, 1, 2, 3, 32, 32), 0)                   # not [R,B,H,2,D,D]
    q, k, v, g, beta = _scan_inputs()
    with pytest.raises(ValueError):
        kda.sp_transition(q, k, v[..., :16], g, beta, None)                 # v width != D
    with pytest.raises(TypeError):
        kda.sp_transition(q, k, v, g, beta, None)                           # host tensors


def test_conv_backward_checks_dy():
    x = torch.zeros(1, 10, 16)
    with pytest.raises(ValueError):
        kda.mshortconv_backward(x, torch.zeros(1, 10, 8), [(kda.MSC_TEXT, 0, 1, 1, 10, 0)], 4,
                                torch.zeros(1, 16, 4))
    with pytest.raises(ValueError):
        kda.mshortconv_backward(x, torch.zeros(1, 10, 16, dtype=torch.bfloat16),
                                [(kda.MSC_TEXT, 0, 1, 1, 10, 0)], 4, torch.zeros(1, 16, 4))
