"""GPU parity of kda_backward against the fp64 oracle's kda_backward, through the C ABI
binding.

The kernel computes in fp32 whatever the input dtype, so every gradient is held to the
fp32 bound (max |gpu - oracle| <= 1e-4 * max |oracle| per (b, h)), with the oracle fed
the same stored (bf16 or fp32) inputs.  Cases: ragged chunk tails, S0 and dS_T given
or absent, Dk != Dv, bf16 and fp32 inputs and output gradients, and the video-clip shape
(B 1, T 32768, H 16, d 128) on two sampled heads.
"""
import numpy as np
import pytest
import torch

from linear_attention_sequence_mshortconv_b200 import kda
from oracle import oracle as O
from tests.parity import compare, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"
GRADS = ("dq", "dk", "dv", "dg", "dbeta")


def _inputs(B, T, H, Dk, Dv, dtype, seed, g_hi=0.1, with_state=True):
    gen = torch.Generator().manual_seed(seed)
    f = dict(generator=gen, dtype=torch.float32)
    unit = lambda z: z / torch.linalg.vector_norm(z, dim=-1, keepdim=True)
    q, k = unit(torch.randn(B, T, H, Dk, **f)), unit(torch.randn(B, T, H, Dk, **f))
    v = torch.randn(B, T, H, Dv, **f)
    g = -(0.001 + (g_hi - 0.001) * torch.rand(B, T, H, Dk, **f))
    beta = torch.sigmoid(torch.randn(B, T, H, **f))
    do = torch.randn(B, T, H, Dv, **f)
    inp = {n: t.to(dtype) for n, t in dict(q=q, k=k, v=v, g=g, beta=beta, do=do).items()}
    S0 = torch.randn(B, H, Dk, Dv, **f) * 0.3 if with_state else None
    dST = torch.randn(B, H, Dk, Dv, **f) * 0.3 if with_state else None
    return inp, S0, dST


def _gpu(inp, S0, dST, do_dtype=None):
    t = {n: x.to(DEV) for n, x in inp.items()}
    do = t["do"] if do_dtype is None else t["do"].to(do_dtype)
    res = kda.backward(t["q"], t["k"], t["v"], t["g"], t["beta"], do,
                       None if S0 is None else S0.to(DEV), None if dST is None else dST.to(DEV))
    torch.cuda.synchronize()
    assert kda.last_device_error() == 0
    return [None if r is None else to_np(r) for r in res]


def _check(inp, S0, dST, heads=None, do_dtype=None):
    got = _gpu(inp, S0, dST, do_dtype)
    do_ref = inp["do"] if do_dtype is None else inp["do"].to(do_dtype)
    B, T, H, _ = inp["q"].shape
    heads = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for (b, h) in heads:
        sl = lambda x: x[b:b + 1, :, h:h + 1].contiguous()
        ref = O.kda_backward(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["g"]), sl(inp["beta"]), sl(do_ref),
                             None if S0 is None else S0[b:b + 1, h:h + 1].double().numpy(),
                             None if dST is None else dST[b:b + 1, h:h + 1].double().numpy())
        for name, gv, rv in zip(GRADS, got[:5], ref[:5]):
            compare(gv[b, :, h], rv[0, :, 0], "fp32", f"{name} b={b} h={h}")
        compare(got[5][b, h], ref[5][0, 0], "fp32", f"dS0 b={b} h={h}")


def test_backward_fp32_small_ragged():
    inp, S0, dST = _inputs(1, 70, 2, 32, 32, torch.float32, seed=31)
    _check(inp, S0, dST)


def test_backward_fp32_dk_ne_dv_no_state():
    inp, _, _ = _inputs(2, 45, 1, 64, 128, torch.float32, seed=32, with_state=False)
    _check(inp, None, None)


def test_backward_bf16_d128():
    inp, S0, dST = _inputs(2, 200, 2, 128, 128, torch.bfloat16, seed=33)
    _check(inp, S0, dST)


def test_backward_bf16_inputs_fp32_output_grad():
    inp, S0, dST = _inputs(1, 96, 3, 128, 64, torch.bfloat16, seed=34)
    inp["do"] = inp["do"].float()
    _check(inp, S0, dST)


def test_backward_single_token_and_exact_chunk():
    for T in (1, 32):
        inp, S0, dST = _inputs(1, T, 1, 32, 32, torch.float32, seed=35 + T)
        _check(inp, S0, dST)


def test_backward_video_clip_shape_sampled_heads():
    inp, _, _ = _inputs(1, 32768, 16, 128, 128, torch.bfloat16, seed=36, with_state=False)
    _check(inp, None, None, heads=[(0, 0), (0, 15)])


def test_backward_near_the_decay_limit():
    """One key channel decays by 2.4 per token (76.8 per 32-token chunk, just inside the
    factorisation's domain of 80) beside gentle channels: still within the fp32 bound."""
    inp, S0, dST = _inputs(1, 100, 2, 32, 32, torch.float32, seed=31)
    inp["g"][:, :, :, 3] = -2.4
    _check(inp, S0, dST)


def test_backward_reports_decay_outside_its_domain():
    """A chunk whose decay on one channel is 96 (3 per token) is outside the domain: the
    call runs, kda_last_device_error() reports KDA_ERR_UNSUPPORTED once and is then clear."""
    inp, S0, dST = _inputs(1, 80, 1, 32, 32, torch.float32, seed=32)
    inp["g"][:, 32:64, :, 5] = -3.0
    t = {n: x.to(DEV) for n, x in inp.items()}
    kda.backward(t["q"], t["k"], t["v"], t["g"], t["beta"], t["do"], S0.to(DEV), dST.to(DEV))
    torch.cuda.synchronize()
    assert kda.last_device_error() == 2   # KDA_ERR_UNSUPPORTED
    assert kda.last_device_error() == 0
    inp["g"][:, 32:64, :, 5] = -2.0       # 64 per chunk: inside
    t = {n: x.to(DEV) for n, x in inp.items()}
    kda.backward(t["q"], t["k"], t["v"], t["g"], t["beta"], t["do"], S0.to(DEV), dST.to(DEV))
    torch.cuda.synchronize()
    assert kda.last_device_error() == 0


def test_backward_empty_sequence_passes_dST_through():
    B, H, D = 1, 2, 32
    z = torch.empty(B, 0, H, D, device=DEV)
    dST = torch.randn(B, H, D, D, device=DEV)
    res = kda.backward(z, z, z, z, torch.empty(B, 0, H, device=DEV), z, None, dST)
    torch.cuda.synchronize()
    assert torch.equal(res[5], dST)
