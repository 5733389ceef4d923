"""GPU parity of kda_forward_varlen (packed samples, state reset at every sample start)
against the fp64 oracle, through the C ABI binding.

Covers empty samples, one-token samples, samples of exactly one chunk, ragged tails
inside the packed axis (a chunk that runs past its sample's end must not touch the next
sample's outputs), per-sample S0, samples long enough to be split into several segments
(state pass + combine per sample), and the CUDA-core path (fp32).
"""
import numpy as np
import pytest
import torch

from linear_attention_sequence_mshortconv_b200 import kda
from oracle import oracle as O
from tests.parity import compare, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _packed(T, H, Dk, Dv, dtype, seed, g_hi=0.1):
    gen = torch.Generator().manual_seed(seed)
    f = dict(generator=gen, dtype=torch.float32)
    unit = lambda z: z / torch.linalg.vector_norm(z, dim=-1, keepdim=True)
    q, k = unit(torch.randn(T, H, Dk, **f)), unit(torch.randn(T, H, Dk, **f))
    v = torch.randn(T, H, Dv, **f)
    g = -(0.001 + (g_hi - 0.001) * torch.rand(T, H, Dk, **f))
    beta = torch.sigmoid(torch.randn(T, H, **f))
    return {n: t.to(dtype) for n, t in dict(q=q, k=k, v=v, g=g, beta=beta).items()}


def _check(cu, inp, S0, kind, o_dtype=torch.float32, chunk=0):
    t = {n: x.to(DEV) for n, x in inp.items()}
    o, ST = kda.forward_varlen(t["q"], t["k"], t["v"], t["g"], t["beta"], cu,
                               None if S0 is None else S0.to(DEV), chunk=chunk, o_dtype=o_dtype)
    torch.cuda.synchronize()
    assert kda.last_device_error() == 0
    o_ref, S_ref = O.kda_forward_varlen(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], cu, S0)
    og, Sg = to_np(o), to_np(ST)
    H = inp["q"].shape[1]
    for i in range(len(cu) - 1):
        a, b = cu[i], cu[i + 1]
        for h in range(H):
            if b > a:
                compare(og[a:b, h], o_ref[a:b, h], kind, f"o sample {i} ({a}:{b}) h={h}")
            compare(Sg[i, h], S_ref[i, h], kind, f"S_T sample {i} h={h}")
    return o, ST


@pytest.mark.parametrize("o_dtype", [torch.float32, torch.bfloat16])
def test_varlen_mixed_lengths_bf16(o_dtype):
    cu = [0, 37, 37, 200, 264, 700, 701, 765, 830]
    H = 3
    inp = _packed(cu[-1], H, 128, 128, torch.bfloat16, seed=1)
    S0 = torch.randn(len(cu) - 1, H, 128, 128, generator=torch.Generator().manual_seed(2)) * 0.3
    o, ST = _check(cu, inp, S0, "bf16", o_dtype=torch.float32)
    if o_dtype == torch.bfloat16:
        # the bf16 output (TMA stores for whole chunks, masked stores for a sample's ragged
        # last chunk) is the fp32 output rounded to nearest even
        t = {n: x.to(DEV) for n, x in inp.items()}
        o16, ST16 = kda.forward_varlen(t["q"], t["k"], t["v"], t["g"], t["beta"], cu, S0.to(DEV),
                                       o_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        assert torch.equal(o16, o.to(torch.bfloat16)) and torch.equal(ST16, ST)


def test_varlen_long_samples_split_into_segments():
    """Long samples get several segments each (state pass + per-sample combine)."""
    cu = [0, 5000, 8000, 8017, 17000]
    inp = _packed(cu[-1], 4, 128, 128, torch.bfloat16, seed=3, g_hi=0.05)
    _check(cu, inp, None, "bf16")


def test_varlen_zero_state_default_and_single_sample_equals_forward():
    cu = [0, 300]
    inp = _packed(300, 2, 128, 128, torch.bfloat16, seed=4)
    t = {n: x.to(DEV) for n, x in inp.items()}
    o, ST = kda.forward_varlen(t["q"], t["k"], t["v"], t["g"], t["beta"], cu, o_dtype=torch.float32)
    o1, ST1 = kda.forward(*(t[n][None] for n in ("q", "k", "v", "g", "beta")), o_dtype=torch.float32)
    torch.cuda.synchronize()
    o_ref, S_ref = O.kda_forward_varlen(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], cu)
    for h in range(2):
        compare(to_np(o)[:, h], o_ref[:, h], "bf16", f"varlen o h={h}")
        compare(to_np(o1)[0, :, h], o_ref[:, h], "bf16", f"forward o h={h}")


@pytest.mark.parametrize("D,chunk", [(32, 16), (128, 16), (64, 128)])
def test_varlen_fp32_cuda_core_path(D, chunk):
    cu = [0, 5, 5, 40, 41, 64] if chunk == 16 else [0, 5, 5, 140, 141, 300]
    inp = _packed(cu[-1], 2, D, D, torch.float32, seed=5)
    S0 = torch.randn(len(cu) - 1, 2, D, D, generator=torch.Generator().manual_seed(6))
    _check(cu, inp, S0, "fp32", chunk=chunk)


def test_varlen_workspace_and_rejections():
    cu = [0, 100, 100, 300]
    inp = _packed(cu[-1], 2, 128, 128, torch.bfloat16, seed=7)
    t = {n: x.to(DEV) for n, x in inp.items()}
    need = kda.varlen_workspace_size(cu, 2, 128, 128, torch.bfloat16, o_dtype=torch.float32)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=DEV)
    o, _ = kda.forward_varlen(t["q"], t["k"], t["v"], t["g"], t["beta"], cu, workspace=ws, o_dtype=torch.float32)
    torch.cuda.synchronize()
    o_ref, _ = O.kda_forward_varlen(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], cu)
    compare(to_np(o)[:, 0], o_ref[:, 0], "bf16", "varlen with caller workspace")
    if need > 256:
        small = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
        with pytest.raises(kda.KdaError):
            kda.forward_varlen(t["q"], t["k"], t["v"], t["g"], t["beta"], cu, workspace=small, o_dtype=torch.float32)
    with pytest.raises((kda.KdaError, ValueError)):
        kda.forward_varlen(t["q"], t["k"], t["v"], t["g"], t["beta"], [5, 100, 300])
