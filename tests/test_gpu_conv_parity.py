"""GPU parity of mshortconv_forward and of the fused conv -> L2 norm -> KDA path against
the fp64 oracle (through the C ABI binding)."""
import numpy as np
import pytest
import torch

from linear_attention_sequence_mshortconv_b200 import inputs as W
from linear_attention_sequence_mshortconv_b200 import kda
from oracle import oracle as O
from tests.parity import compare, compare_heads, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"
TEXT, IMAGE, VIDEO = 0, 1, 2


def _mixed_segments(gap=False):
    """text 37 | image 9x13 | video 4x5x7 | text 11 | image 3x4 (two weight sets), with an
    optional uncovered gap of 5 tokens before the video."""
    segs, pos = [], 0
    for (m, Fr, Hh, Wd, ws) in [(TEXT, 1, 1, 37, 0), (IMAGE, 1, 9, 13, 0), (VIDEO, 4, 5, 7, 0),
                                (TEXT, 1, 1, 11, 1), (IMAGE, 1, 3, 4, 1)]:
        if gap and m == VIDEO:
            pos += 5
        segs.append((m, pos, Fr, Hh, Wd, ws))
        pos += Wd if m == TEXT else (Hh * Wd if m == IMAGE else Fr * Hh * Wd)
    return segs, pos


def _weights(C, Kt, seed, sets=2):
    gen = torch.Generator().manual_seed(seed)
    return (torch.randn(sets, C, Kt, generator=gen) / Kt ** 0.5,
            torch.randn(sets, C, 3, 3, generator=gen) / 3.0,
            torch.randn(sets, C, 3, 3, 3, generator=gen) / 27 ** 0.5)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("gap", [False, True])
def test_conv_all_modalities(dtype, gap):
    segs, T = _mixed_segments(gap)
    B, C, Kt = 2, 64, 4
    x = torch.randn(B, T, C, generator=torch.Generator().manual_seed(3)).to(dtype)
    wt, wi, wv = _weights(C, Kt, 4)
    y = kda.mshortconv(x.to(DEV), segs, Kt, wt.to(DEV), wi.to(DEV), wv.to(DEV))
    torch.cuda.synchronize()
    ref = O.mshortconv(x, segs, Kt, wt, wi, wv)
    kind = "fp32" if dtype == torch.float32 else "bf16"
    for b in range(B):
        compare(to_np(y)[b], ref[b], kind, f"conv b={b}")


def test_conv_bf16_output_is_the_rounded_fp32_sum():
    """bf16 output must be the fp32 accumulation rounded once: within half a bf16 ulp
    of the fp64 result plus fp32 accumulation error."""
    segs, T = _mixed_segments()
    x = torch.randn(1, T, 16, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    wt, wi, wv = _weights(16, 4, 6)
    y = kda.mshortconv(x.to(DEV), segs, 4, wt.to(DEV), wi.to(DEV), wv.to(DEV)).float().cpu()
    ref = torch.from_numpy(O.mshortconv(x, segs, 4, wt, wi, wv))
    ulp = torch.clamp(ref.abs(), min=1e-30) * 2.0 ** -7   # ulp of bf16 at |ref| is at most |ref| * 2^-7
    assert torch.all((y.double() - ref).abs() <= 0.5 * ulp + 1e-5 * ref.abs().max())


@pytest.mark.parametrize("B", [1, 2])
def test_conv_tiled_path_wide_channels(B):
    """C = 256 (whole 128-channel blocks): image and video segments take the tiled kernel.
    Ragged tiles in both directions, a video long enough for the frame ring to wrap, an
    image that is an exact multiple of the tile, both weight sets, and a text segment
    between visual ones.  bf16 output = the fp32 sum rounded once."""
    segs, pos = [], 0
    for (m, Fr, Hh, Wd, ws) in [(TEXT, 1, 1, 7, 0), (IMAGE, 1, 17, 33, 0), (VIDEO, 7, 11, 19, 1),
                                (TEXT, 1, 1, 5, 1), (IMAGE, 1, 8, 16, 1), (VIDEO, 3, 8, 16, 0)]:
        segs.append((m, pos, Fr, Hh, Wd, ws))
        pos += Wd if m == TEXT else (Hh * Wd if m == IMAGE else Fr * Hh * Wd)
    T, C, Kt = pos, 256, 4
    x = torch.randn(B, T, C, generator=torch.Generator().manual_seed(21)).to(torch.bfloat16)
    wt, wi, wv = _weights(C, Kt, 22)
    y = kda.mshortconv(x.to(DEV), segs, Kt, wt.to(DEV), wi.to(DEV), wv.to(DEV))
    torch.cuda.synchronize()
    assert kda.last_device_error() == 0
    ref = torch.from_numpy(O.mshortconv(x, segs, Kt, wt, wi, wv))
    y = y.float().cpu().double()
    ulp = torch.clamp(ref.abs(), min=1e-30) * 2.0 ** -7
    bad = (y - ref).abs() > 0.5 * ulp + 1e-5 * ref.abs().max()
    assert not bool(bad.any()), f"{int(bad.sum())} elements off, first at {bad.nonzero()[0].tolist()}"


@pytest.mark.parametrize("chunk", [0, 128])
def test_fused_small_mixed_stream(chunk):
    segs, T = _mixed_segments()
    B, H, D, Kt = 1, 2, 128, 4
    C = H * D
    gen = torch.Generator().manual_seed(9)
    xq, xk, xv = (torch.randn(B, T, C, generator=gen).to(torch.bfloat16) for _ in range(3))
    g = (-(0.001 + 0.099 * torch.rand(B, T, H, D, generator=gen))).to(torch.bfloat16)
    beta = torch.sigmoid(torch.randn(B, T, H, generator=gen)).to(torch.bfloat16)
    ws = [tuple(w[:1].contiguous() for w in _weights(C, Kt, s)) for s in (10, 11, 12)]
    segs0 = [(m, s, Fr, Hh, Wd, 0) for (m, s, Fr, Hh, Wd, _) in segs]
    dv = lambda t: t.to(DEV)
    o, ST = kda.mshortconv_kda_forward(dv(xq), dv(xk), dv(xv), segs0, Kt,
                                       [dv(w) for w in ws[0]], [dv(w) for w in ws[1]],
                                       [dv(w) for w in ws[2]], dv(g), dv(beta),
                                       chunk=chunk, o_dtype=torch.float32)
    o16, ST16 = kda.mshortconv_kda_forward(dv(xq), dv(xk), dv(xv), segs0, Kt,
                                           [dv(w) for w in ws[0]], [dv(w) for w in ws[1]],
                                           [dv(w) for w in ws[2]], dv(g), dv(beta), chunk=chunk)
    torch.cuda.synchronize()
    assert torch.equal(o16, o.to(torch.bfloat16)) and torch.equal(ST16, ST)
    o_ref, S_ref = O.fused_forward(xq, xk, xv, segs0, Kt, ws[0], ws[1], ws[2], g, beta, H)
    compare_heads(to_np(o), o_ref, to_np(ST), S_ref, "bf16", what=f"fused small, chunk {chunk}")


def test_fused_full_size_sampled_heads():
    w = W.FUSED_MIXED
    inp = W.make_fused_inputs(w, device=DEV)
    o, ST = kda.mshortconv_kda_forward(inp["xq"], inp["xk"], inp["xv"], inp["segments"], w.Kt,
                                       inp["wq"], inp["wk"], inp["wv"], inp["g"], inp["beta"],
                                       chunk=w.chunk, o_dtype=torch.float32)
    torch.cuda.synchronize()
    assert kda.last_device_error() == 0
    D = w.D
    for h in (0, 11):
        sl = slice(h * D, (h + 1) * D)
        cpu = lambda t: t[:, :, sl].contiguous().cpu()
        wsl = lambda ws: tuple(x[:, sl].contiguous().cpu() for x in ws)
        o_ref, S_ref = O.fused_forward(cpu(inp["xq"]), cpu(inp["xk"]), cpu(inp["xv"]),
                                       inp["segments"], w.Kt, wsl(inp["wq"]), wsl(inp["wk"]),
                                       wsl(inp["wv"]), inp["g"][:, :, h:h + 1].cpu(),
                                       inp["beta"][:, :, h:h + 1].cpu(), 1)
        compare(to_np(o[:, :, h])[0], o_ref[0, :, 0], "bf16", f"fused o h={h}")
        compare(ST[0, h].cpu().numpy(), S_ref[0, 0], "bf16", f"fused S_T h={h}")
