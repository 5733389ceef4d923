"""GPU parity of mshortconv_backward against the fp64 oracle's mshortconv_backward,
through the C ABI binding.

Streams mix text (Kt = 4), image and video segments with gaps that no segment covers
(dx must be 0 there), fp32 and bf16 inputs, a channel count that is not a multiple of
32, several weight sets per modality, and a stream with the fused workload's segment
shapes at reduced channel count.  Gradients are fp32 on both sides: max |gpu - oracle|
<= 1e-4 * max |oracle| for dx and for each weight gradient.
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


def _case(segs, T, B, C, dtype, seed, Kt=4, sets=(1, 2, 1)):
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn(B, T, C, generator=gen).to(dtype)
    dy = torch.randn(B, T, C, generator=gen).to(dtype)
    wt = torch.randn(sets[0], C, Kt, generator=gen) / 2
    wi = torch.randn(sets[1], C, 3, 3, generator=gen) / 3
    wv = torch.randn(sets[2], C, 3, 3, 3, generator=gen) / 5
    got = kda.mshortconv_backward(x.to(DEV), dy.to(DEV), segs, Kt, wt.to(DEV), wi.to(DEV), wv.to(DEV))
    torch.cuda.synchronize()
    ref = O.mshortconv_backward(x, dy, segs, Kt, wt, wi, wv)
    for name, gv, rv in zip(("dx", "dw_text", "dw_image", "dw_video"), got, ref):
        compare(to_np(gv), rv, "fp32", name)
    return got, ref


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_conv_backward_mixed_stream(dtype):
    segs = [(TEXT, 0, 1, 1, 37, 0), (IMAGE, 40, 1, 9, 11, 1), (VIDEO, 139, 4, 6, 7, 0), (IMAGE, 307, 1, 5, 4, 0)]
    T = 330
    got, _ = _case(segs, T, 2, 64, dtype, seed=41)
    dx = to_np(got[0])
    for a, b in ((37, 40), (139 + 168, 307), (327, 330)):
        assert np.all(dx[:, a:b] == 0.0)


def test_conv_backward_channels_not_multiple_of_32():
    segs = [(TEXT, 0, 1, 1, 20, 0), (VIDEO, 20, 3, 5, 6, 0)]
    _case(segs, 110, 1, 40, torch.bfloat16, seed=42)


def test_conv_backward_fused_workload_shapes():
    # 512 text + 64x64 image + 8x32x48 video (the fused stream with fewer frames), C = 256
    segs = [(TEXT, 0, 1, 1, 512, 0), (IMAGE, 512, 1, 64, 64, 0), (VIDEO, 4608, 8, 32, 48, 0)]
    _case(segs, 4608 + 8 * 32 * 48, 1, 256, torch.bfloat16, seed=43, sets=(1, 1, 1))
