"""Pins of the oracle's mShortConv backward (mshortconv_backward) to things other than
itself.

* Library routine: torch.autograd through torch.nn.functional.conv1d / conv2d / conv3d
  in fp64 (groups = C, the zero pads of section 3.4) on every segment gives dx and the
  weight gradients.
* Adjoint identities with the (separately pinned) forward oracle: y = conv(x; w) is
  linear in x and in w, so sum(dy * y) = sum(x * dx) = sum(w * dw) for each modality.
* Tokens covered by no segment get dx = 0.
"""
import numpy as np
import torch
import torch.nn.functional as Fn

from oracle import oracle as O

TEXT, IMAGE, VIDEO = O.MOD_TEXT, O.MOD_IMAGE, O.MOD_VIDEO
KT = 4
# text 7 | gap 2 | image 5x6 | video 3x4x5 | gap 3   (T = 7 + 2 + 30 + 60 + 3 = 102)
SEGS = [(TEXT, 0, 1, 1, 7, 0), (IMAGE, 9, 1, 5, 6, 1), (VIDEO, 39, 3, 4, 5, 0)]
T = 102


def _inputs(B=2, C=8, seed=0):
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn(B, T, C, generator=gen, dtype=torch.float64)
    dy = torch.randn(B, T, C, generator=gen, dtype=torch.float64)
    wt = torch.randn(1, C, KT, generator=gen, dtype=torch.float64)
    wi = torch.randn(2, C, 3, 3, generator=gen, dtype=torch.float64)
    wv = torch.randn(1, C, 3, 3, 3, generator=gen, dtype=torch.float64)
    return x, dy, wt, wi, wv


def test_conv_backward_matches_torch_autograd():
    x, dy, wt, wi, wv = _inputs()
    B, _, C = x.shape
    dx, dwt, dwi, dwv = O.mshortconv_backward(x, dy, SEGS, KT, wt, wi, wv)
    xl = x.clone().requires_grad_(True)
    wl = [w.clone().requires_grad_(True) for w in (wt, wi, wv)]
    loss = 0.0
    for (m, s, F, Hh, Wd, ws) in SEGS:
        if m == TEXT:
            xs = xl[:, s:s + Wd].permute(0, 2, 1)                              # [B, C, L]
            y = Fn.conv1d(Fn.pad(xs, (KT - 1, 0)), wl[0][ws].view(C, 1, KT), groups=C)
            loss = loss + (y * dy[:, s:s + Wd].permute(0, 2, 1)).sum()
        elif m == IMAGE:
            n = Hh * Wd
            xs = xl[:, s:s + n].reshape(B, Hh, Wd, C).permute(0, 3, 1, 2)
            y = Fn.conv2d(Fn.pad(xs, (1, 1, 1, 1)), wl[1][ws].view(C, 1, 3, 3), groups=C)
            loss = loss + (y * dy[:, s:s + n].reshape(B, Hh, Wd, C).permute(0, 3, 1, 2)).sum()
        else:
            n = F * Hh * Wd
            xs = xl[:, s:s + n].reshape(B, F, Hh, Wd, C).permute(0, 4, 1, 2, 3)
            y = Fn.conv3d(Fn.pad(xs, (1, 1, 1, 1, 2, 0)), wl[2][ws].view(C, 1, 3, 3, 3), groups=C)
            loss = loss + (y * dy[:, s:s + n].reshape(B, F, Hh, Wd, C).permute(0, 4, 1, 2, 3)).sum()
    loss.backward()
    assert np.abs(dx - xl.grad.numpy()).max() <= 1e-12 * np.abs(dx).max()
    for got, leaf in zip((dwt, dwi, dwv), wl):
        ref = leaf.grad.numpy()
        assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())
    # uncovered tokens
    for a, b in ((7, 9), (99, 102)):
        assert np.all(dx[:, a:b] == 0.0)


def test_conv_backward_adjoint_identities():
    x, dy, wt, wi, wv = _inputs(seed=1)
    dx, dwt, dwi, dwv = O.mshortconv_backward(x, dy, SEGS, KT, wt, wi, wv)
    y = O.mshortconv(x, SEGS, KT, wt.float(), wi.float(), wv.float())
    # the forward oracle reads the fp32 weights; use those same values on the adjoint side
    dx32, dwt32, dwi32, dwv32 = O.mshortconv_backward(x, dy, SEGS, KT, wt.float(), wi.float(), wv.float())
    lhs = float((y * dy.numpy()).sum())
    assert abs(lhs - float((x.numpy() * dx32).sum())) <= 1e-11 * abs(lhs)
    wsum = sum(float((w.float().double().numpy() * d).sum()) for w, d in ((wt, dwt32), (wi, dwi32), (wv, dwv32)))
    assert abs(lhs - wsum) <= 1e-11 * abs(lhs)
