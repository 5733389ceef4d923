"""Pins of the oracle's fused backward (fused_backward) and the norm's backward
(l2norm_heads_backward) to things other than themselves: torch.autograd through an fp64
implementation of the whole fused forward written here (torch conv1d/2d/3d with the
segment pads, torch.nn.functional.normalize per head, the token loop of Eq. 14), and
through normalize alone, including an all-zero head slice."""
import numpy as np
import torch
import torch.nn.functional as Fn

from oracle import oracle as O

TEXT, IMAGE, VIDEO = O.MOD_TEXT, O.MOD_IMAGE, O.MOD_VIDEO
KT = 4
SEGS = [(TEXT, 0, 1, 1, 6, 0), (IMAGE, 6, 1, 3, 4, 0), (VIDEO, 18, 3, 2, 3, 0)]
T = 18 + 18 + 2   # two trailing tokens outside every segment


def _conv(x, w3, C):
    B = x.shape[0]
    y = torch.zeros_like(x)
    for (m, s, F, Hh, Wd, ws) in SEGS:
        if m == TEXT:
            xs = x[:, s:s + Wd].permute(0, 2, 1)
            ys = Fn.conv1d(Fn.pad(xs, (KT - 1, 0)), w3[0][ws].view(C, 1, KT), groups=C).permute(0, 2, 1)
            y = torch.cat([y[:, :s], ys, y[:, s + Wd:]], dim=1)
        elif m == IMAGE:
            n = Hh * Wd
            xs = x[:, s:s + n].reshape(B, Hh, Wd, C).permute(0, 3, 1, 2)
            ys = Fn.conv2d(Fn.pad(xs, (1, 1, 1, 1)), w3[1][ws].view(C, 1, 3, 3), groups=C)
            y = torch.cat([y[:, :s], ys.permute(0, 2, 3, 1).reshape(B, n, C), y[:, s + n:]], dim=1)
        else:
            n = F * Hh * Wd
            xs = x[:, s:s + n].reshape(B, F, Hh, Wd, C).permute(0, 4, 1, 2, 3)
            ys = Fn.conv3d(Fn.pad(xs, (1, 1, 1, 1, 2, 0)), w3[2][ws].view(C, 1, 3, 3, 3), groups=C)
            y = torch.cat([y[:, :s], ys.permute(0, 2, 3, 4, 1).reshape(B, n, C), y[:, s + n:]], dim=1)
    return y


def _scan(q, k, v, g, beta, S0):
    B, Tn, H, D = q.shape
    outs, fins = [], []
    for b in range(B):
        ob, fb = [], []
        for h in range(H):
            S = S0[b, h]
            oh = []
            for t in range(Tn):
                kk = k[b, t, h]
                S = torch.exp(g[b, t, h])[:, None] * S
                S = S - beta[b, t, h] * torch.outer(kk, kk @ S) + beta[b, t, h] * torch.outer(kk, v[b, t, h])
                oh.append(S.T @ q[b, t, h])
            ob.append(torch.stack(oh))
            fb.append(S)
        outs.append(torch.stack(ob, dim=1))
        fins.append(torch.stack(fb))
    return torch.stack(outs), torch.stack(fins)


def test_fused_backward_matches_autograd_of_the_fused_forward():
    B, H, D = 1, 2, 4
    C = H * D
    gen = torch.Generator().manual_seed(5)
    r = lambda *s: torch.randn(*s, generator=gen, dtype=torch.float64)
    xq, xk, xv = r(B, T, C), r(B, T, C), r(B, T, C)
    # weights exactly representable in fp32 (the forward oracle stores weights as fp32)
    ws = [tuple(w.float().double() for w in (r(1, C, KT) / 2, r(1, C, 3, 3) / 3, r(1, C, 3, 3, 3) / 5))
          for _ in range(3)]
    g = -torch.rand(B, T, H, D, generator=gen, dtype=torch.float64) * 0.3
    beta = torch.rand(B, T, H, generator=gen, dtype=torch.float64)
    S0, dST, do = r(B, H, D, D) * 0.3, r(B, H, D, D), r(B, T, H, D)
    leaves = [t.clone().requires_grad_(True) for t in (xq, xk, xv, g, beta, S0)]
    wl = [tuple(w.clone().requires_grad_(True) for w in ws3) for ws3 in ws]
    lq, lk, lv, lg, lb, lS = leaves
    nq = Fn.normalize(_conv(lq, wl[0], C).reshape(B, T, H, D), dim=-1, eps=1e-300)
    nk = Fn.normalize(_conv(lk, wl[1], C).reshape(B, T, H, D), dim=-1, eps=1e-300)
    vv = _conv(lv, wl[2], C).reshape(B, T, H, D)
    o, S = _scan(nq, nk, vv, lg, lb, lS)
    ((o * do).sum() + (S * dST).sum()).backward()
    w32 = [tuple(w.numpy() for w in ws3) for ws3 in ws]   # fp64 arrays, read exactly
    got = O.fused_backward(xq, xk, xv, SEGS, KT, w32[0], w32[1], w32[2], g, beta, H, do, S0.numpy(), dST.numpy())
    dxq, dxk, dxv, dwq, dwk, dwv, dg, dbeta, dS0 = got
    for mine, leaf in zip((dxq, dxk, dxv, dg, dbeta, dS0), leaves):
        ref = leaf.grad.numpy()
        assert np.abs(mine - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max())
    for mine3, leaf3 in zip((dwq, dwk, dwv), wl):
        for mine, leaf in zip(mine3, leaf3):
            ref = leaf.grad.numpy()
            assert np.abs(mine - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max())


def test_l2norm_backward_matches_autograd_and_zero_slices():
    gen = torch.Generator().manual_seed(6)
    x = torch.randn(3, 5, 2 * 6, generator=gen, dtype=torch.float64)
    x[1, 2, 6:] = 0.0                                   # an all-zero head slice
    dy = torch.randn(3, 5, 12, generator=gen, dtype=torch.float64)
    got = O.l2norm_heads_backward(x, dy, 2)
    xl = x.clone().requires_grad_(True)
    y = Fn.normalize(xl.reshape(3, 5, 2, 6), dim=-1, eps=1e-300).reshape(3, 5, 12)
    (y * dy).sum().backward()
    ref = xl.grad.numpy()
    mask = np.ones_like(ref, dtype=bool)
    mask[1, 2, 6:] = False
    assert np.abs(got[mask] - ref[mask]).max() <= 1e-12 * np.abs(ref).max()
    assert np.all(got[1, 2, 6:] == 0.0)
