"""GPU parity of kda_forward_gated (the output side of Eq. 15: Sigmoid(gate) * gamma *
RMSNorm(S_t^T q_t)) against the fp64 oracle, through the C ABI binding.

Paths: the CUDA-core scan + the epilogue kernel (fp32 inputs, other head widths), the
tensor-core scan + the epilogue kernel (fp32 output) and the tensor-core scan with the
epilogue fused into its output stage (bf16 output).  Tolerances: fp32 inputs 1e-4 of
max|ref| per (b, h); bf16 inputs 2e-2 of RMS(ref) per (b, h), plus, for a bf16 output,
the rounding of y itself (2^-8 |ref|: the outputs are heavy-tailed).
"""
import numpy as np
import pytest
import torch

from linear_attention_sequence_mshortconv_b200 import inputs as W
from linear_attention_sequence_mshortconv_b200 import kda
from oracle import oracle as O
from tests.parity import compare, to_np
from tests.test_gpu_kda_parity import _custom

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gate_gamma(B, T, H, Dv, dtype, seed):
    gen = torch.Generator().manual_seed(seed)
    gate = torch.randn(B, T, H, Dv, generator=gen).to(dtype)
    gamma = 0.5 + torch.rand(H, Dv, generator=gen)
    return gate, gamma


def _run(inp, gate, gamma, eps, o_dtype, chunk=0):
    t = {k: v.to(DEV) for k, v in inp.items() if isinstance(v, torch.Tensor)}
    y, ST = kda.forward_gated(t["q"], t["k"], t["v"], t["g"], t["beta"], gate.to(DEV),
                              None if gamma is None else gamma.to(DEV), eps, chunk=chunk, o_dtype=o_dtype)
    torch.cuda.synchronize()
    assert kda.last_device_error() == 0
    return to_np(y), to_np(ST)


def _check(y, y_ref, ST, S_ref, kind, bf16_out, what):
    B, T, H, _ = y_ref.shape
    for b in range(B):
        for h in range(H):
            r = y_ref[b, :, h]
            if kind == "bf16":
                bound = 2e-2 * np.sqrt(np.mean(r * r)) + (2.0 ** -8 * np.abs(r) if bf16_out else 0.0)
                err = np.abs(y[b, :, h] - r)
                assert np.all(err <= bound), f"{what} y[b={b},h={h}] worst excess {np.max(err - bound):.3e}"
            else:
                compare(y[b, :, h], r, "fp32", f"{what} y[b={b},h={h}]")
            compare(ST[b, h], S_ref[b, h], kind, f"{what} S_T[b={b},h={h}]")


def test_gated_tiny_fp32():
    w = W.TINY_FP32
    inp = W.make_kda_inputs(w)
    gate, gamma = _gate_gamma(w.B, w.T, w.H, w.D, torch.float32, 1)
    y, ST = _run(inp, gate, gamma, 1e-6, torch.float32, chunk=w.chunk)
    y_ref, S_ref = O.kda_forward_gated(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], gate, gamma, 1e-6)
    _check(y, y_ref, ST, S_ref, "fp32", False, "tiny fp32")


@pytest.mark.parametrize("o_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,T,H,D", [(2, 300, 3, 128), (1, 64, 2, 128), (1, 97, 2, 64)])
@pytest.mark.parametrize("with_gamma", [True, False])
def test_gated_bf16_paths(o_dtype, B, T, H, D, with_gamma):
    inp = _custom(B, T, H, D, D, torch.bfloat16, seed=T + H)
    gate, gamma = _gate_gamma(B, T, H, D, torch.bfloat16, T)
    gamma = gamma if with_gamma else None
    y, ST = _run(inp, gate, gamma, 1e-5, o_dtype)
    y_ref, S_ref = O.kda_forward_gated(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], gate, gamma, 1e-5)
    _check(y, y_ref, ST, S_ref, "bf16", o_dtype == torch.bfloat16, f"B{B} T{T} H{H} D{D}")


@pytest.mark.parametrize("dtype,T,D", [(torch.float32, 200, 64), (torch.bfloat16, 150, 128)])
def test_gated_chunk_128(dtype, T, D):
    """128-token chunks (the CUDA-core scan) followed by the epilogue kernel."""
    inp = _custom(1, T, 2, D, D, dtype, seed=T + D)
    gate, gamma = _gate_gamma(1, T, 2, D, dtype, T)
    y, ST = _run(inp, gate, gamma, 1e-6, torch.float32, chunk=128)
    y_ref, S_ref = O.kda_forward_gated(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], gate, gamma, 1e-6)
    _check(y, y_ref, ST, S_ref, "fp32" if dtype == torch.float32 else "bf16", False, f"chunk 128 {dtype} D{D}")


def test_gated_ungated_readout_unchanged():
    """The plain scan's output is untouched by the gated path: with the gate wide open
    and gamma = 1, eps = 0, the gated output is the plain readout divided by its RMS."""
    inp = _custom(1, 200, 2, 128, 128, torch.bfloat16, seed=5)
    t = {k: v.to(DEV) for k, v in inp.items() if isinstance(v, torch.Tensor)}
    o, _ = kda.forward(t["q"], t["k"], t["v"], t["g"], t["beta"], o_dtype=torch.float32)
    gate = torch.full((1, 200, 2, 128), 30.0, dtype=torch.bfloat16, device=DEV)
    y, _ = kda.forward_gated(t["q"], t["k"], t["v"], t["g"], t["beta"], gate, None, 0.0, o_dtype=torch.float32)
    torch.cuda.synchronize()
    o, y = o.double(), y.double()
    rms = torch.sqrt(torch.mean(o * o, dim=-1, keepdim=True))
    assert torch.allclose(y, o / rms, rtol=1e-4, atol=1e-5)


def test_gated_video_clip_full_size_sampled_head():
    w = W.VIDEO_CLIP
    inp = W.make_kda_inputs(w, device=DEV)
    gate, gamma = _gate_gamma(w.B, w.T, w.H, w.D, torch.bfloat16, 42)
    y, ST = kda.forward_gated(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], gate.to(DEV),
                              gamma.to(DEV), 1e-6, chunk=w.chunk, o_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert kda.last_device_error() == 0
    h = 7
    cpu = {k: v[:, :, h:h + 1].contiguous().cpu() for k, v in inp.items() if isinstance(v, torch.Tensor)}
    y_ref, S_ref = O.kda_forward_gated(cpu["q"], cpu["k"], cpu["v"], cpu["g"], cpu["beta"],
                                       gate[:, :, h:h + 1].contiguous(), gamma[h:h + 1], 1e-6)
    _check(to_np(y[:, :, h:h + 1]), y_ref, to_np(ST[:, h:h + 1]), S_ref, "bf16", True, "video clip gated")
