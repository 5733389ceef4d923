"""GPU parity of kda_mshortconv_backward (the fused conv -> per-head norm -> scan path)
against the fp64 oracle's fused_backward, through the C ABI binding.

The CUDA path widens bf16 inputs exactly and runs the chain rule in fp32, so every
gradient is held to the fp32 bound (max |gpu - oracle| <= 1e-4 * max |oracle|).  Streams
mix text, image and video segments and trailing tokens outside every segment.
"""
import numpy as np
import pytest
import torch

from linear_attention_sequence_mshortconv_b200 import kda
from oracle import oracle as O
from tests.parity import compare, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"
TEXT, IMAGE, VIDEO = kda.MSC_TEXT, kda.MSC_IMAGE, kda.MSC_VIDEO


def _case(segs, T, B, H, D, dtype, seed, Kt=4):
    C = H * D
    gen = torch.Generator().manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=gen)
    xq, xk, xv = (r(B, T, C).to(dtype) for _ in range(3))
    ws = [(r(1, C, Kt) / 2, r(1, C, 3, 3) / 3, r(1, C, 3, 3, 3) / 5) for _ in range(3)]
    g = (-(0.001 + 0.099 * torch.rand(B, T, H, D, generator=gen))).to(dtype)
    beta = torch.sigmoid(r(B, T, H)).to(dtype)
    do = r(B, T, H, D).to(dtype)
    S0, dST = r(B, H, D, D) * 0.3, r(B, H, D, D) * 0.3
    d = lambda t: t.to(DEV)
    got = kda.mshortconv_kda_backward(d(xq), d(xk), d(xv), segs, Kt, [d(w) for w in ws[0]], [d(w) for w in ws[1]],
                                      [d(w) for w in ws[2]], d(g), d(beta), d(do), d(S0), d(dST))
    torch.cuda.synchronize()
    assert kda.last_device_error() == 0
    ref = O.fused_backward(xq, xk, xv, segs, Kt, ws[0], ws[1], ws[2], g, beta, H, do, S0.double().numpy(),
                           dST.double().numpy())
    dxq, dxk, dxv, dwq, dwk, dwv, dg, dbeta, dS0 = ref
    for name, rv in (("dxq", dxq), ("dxk", dxk), ("dxv", dxv), ("dg", dg), ("dbeta", dbeta), ("dS0", dS0)):
        compare(to_np(got[name]), rv, "fp32", name)
    for name, rv3 in (("dwq", dwq), ("dwk", dwk), ("dwv", dwv)):
        for m, rv in enumerate(rv3):
            compare(to_np(got[name][m]), rv, "fp32", f"{name}[{m}]")


def test_fused_backward_bf16_d128():
    segs = [(TEXT, 0, 1, 1, 40, 0), (IMAGE, 40, 1, 8, 10, 0), (VIDEO, 120, 3, 6, 7, 0)]
    _case(segs, 250, 1, 2, 128, torch.bfloat16, seed=51)


def test_fused_backward_fp32_d32_two_rows():
    segs = [(TEXT, 0, 1, 1, 17, 0), (VIDEO, 17, 2, 3, 5, 0), (IMAGE, 47, 1, 4, 4, 0)]
    _case(segs, 66, 2, 2, 32, torch.float32, seed=52)
