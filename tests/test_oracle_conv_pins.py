"""Pins for the oracle's modality-aware short convolution (Chimera paper, section 3.4,
pchao.org translation; the agifrontier summary adds "causal in time, symmetric in
space" and the 2-D treatment of an image).

The conv is depthwise, restarts at every segment, is causal 1-D for text, 3x3 spatial
for an image and 3x3x3 (causal in time, symmetric in space) for video, with the
visual tokens in the time-first raster order of Eq. 12.  These tests pin the oracle
to PyTorch's own conv1d/conv2d/conv3d (a library routine, fp64 on the CPU, groups=C,
explicit zero padding per segment) and to closed-form responses.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import oracle as O

TEXT, IMAGE, VIDEO = O.MOD_TEXT, O.MOD_IMAGE, O.MOD_VIDEO


def _segments():
    # text 37 | image 9x13 (set 0) | video 4x5x7 (set 0) | text 11 (set 1) | image 3x4 (set 1)
    segs, pos = [], 0
    for (m, Fr, Hh, W, ws) in [(TEXT, 1, 1, 37, 0), (IMAGE, 1, 9, 13, 0), (VIDEO, 4, 5, 7, 0),
                               (TEXT, 1, 1, 11, 1), (IMAGE, 1, 3, 4, 1)]:
        segs.append((m, pos, Fr, Hh, W, ws))
        pos += W if m == TEXT else (Hh * W if m == IMAGE else Fr * Hh * W)
    return segs, pos


def _weights(rng, C, Kt):
    return (rng.standard_normal((2, C, Kt)).astype(np.float32),
            rng.standard_normal((2, C, 3, 3)).astype(np.float32),
            rng.standard_normal((1, C, 3, 3, 3)).astype(np.float32))


def _torch_reference(x, segs, Kt, wt, wi, wv):
    """Per-segment depthwise conv with torch.nn.functional in float64."""
    B, T, C = x.shape
    y = np.zeros_like(x)
    X = torch.from_numpy(x)
    for (m, s, Fr, Hh, W, ws) in segs:
        if m == TEXT:
            seg = X[:, s:s + W].permute(0, 2, 1)                        # [B,C,L]
            w = torch.from_numpy(wt[ws]).double().unsqueeze(1)           # [C,1,Kt]
            out = F.conv1d(F.pad(seg, (Kt - 1, 0)), w, groups=C)
            y[:, s:s + W] = out.permute(0, 2, 1).numpy()
        elif m == IMAGE:
            n = Hh * W
            seg = X[:, s:s + n].permute(0, 2, 1).reshape(B, C, Hh, W)
            w = torch.from_numpy(wi[ws]).double().unsqueeze(1)           # [C,1,3,3]
            out = F.conv2d(seg, w, padding=1, groups=C)
            y[:, s:s + n] = out.reshape(B, C, n).permute(0, 2, 1).numpy()
        else:
            n = Fr * Hh * W
            seg = X[:, s:s + n].permute(0, 2, 1).reshape(B, C, Fr, Hh, W)
            w = torch.from_numpy(wv[ws]).double().unsqueeze(1)           # [C,1,3,3,3]
            out = F.conv3d(F.pad(seg, (1, 1, 1, 1, 2, 0)), w, groups=C)  # causal in time
            y[:, s:s + n] = out.reshape(B, C, n).permute(0, 2, 1).numpy()
    return y


@pytest.mark.parametrize("Kt", [4, 2])
def test_conv_matches_torch_conv_routines(Kt):
    rng = np.random.default_rng(Kt)
    segs, T = _segments()
    B, C = 2, 6
    x = rng.standard_normal((B, T, C))
    wt, wi, wv = _weights(rng, C, Kt)
    y = O.mshortconv(x, segs, Kt, wt, wi, wv)
    ref = _torch_reference(x, segs, Kt, wt, wi, wv)
    assert np.abs(y - ref).max() <= 1e-12


def test_conv_channel_range_and_bf16_input():
    rng = np.random.default_rng(1)
    segs, T = _segments()
    B, C = 1, 8
    xt = torch.from_numpy(rng.standard_normal((B, T, C)).astype(np.float32)).to(torch.bfloat16)
    wt, wi, wv = _weights(rng, C, 4)
    full = O.mshortconv(xt, segs, 4, wt, wi, wv)
    part = O.mshortconv(xt, segs, 4, wt, wi, wv, c_range=(3, 6))
    assert np.array_equal(part, full[:, :, 3:6])
    ref = _torch_reference(xt.double().numpy(), segs, 4, wt, wi, wv)
    assert np.abs(full - ref).max() <= 1e-12


def test_impulse_response_reproduces_kernels():
    C, Kt = 1, 4
    rng = np.random.default_rng(2)
    wt, wi, wv = _weights(rng, C, Kt)
    # text: a delta at t0 appears as w[j] at t0 + (Kt-1) - j
    L, t0 = 12, 5
    x = np.zeros((1, L, C)); x[0, t0, 0] = 1.0
    y = O.mshortconv(x, [(TEXT, 0, 1, 1, L, 0)], Kt, wt, wi, wv)[0, :, 0]
    expect = np.zeros(L)
    for j in range(Kt):
        expect[t0 + (Kt - 1) - j] = wt[0, 0, j]
    assert np.abs(y - expect).max() == 0.0
    # image: a delta at (r0, c0) appears as w[a,e] at (r0+1-a, c0+1-e)
    Hh, W, r0, c0 = 5, 6, 2, 3
    x = np.zeros((1, Hh * W, C)); x[0, r0 * W + c0, 0] = 1.0
    y = O.mshortconv(x, [(IMAGE, 0, 1, Hh, W, 0)], Kt, wt, wi, wv)[0, :, 0].reshape(Hh, W)
    expect = np.zeros((Hh, W))
    for a in range(3):
        for e in range(3):
            expect[r0 + 1 - a, c0 + 1 - e] = wi[0, 0, a, e]
    assert np.abs(y - expect).max() == 0.0
    # video: a delta at frame f0 reaches frames f0, f0+1, f0+2 only (causal in time)
    Fr, f0 = 5, 1
    x = np.zeros((1, Fr * Hh * W, C)); x[0, (f0 * Hh + r0) * W + c0, 0] = 1.0
    y = O.mshortconv(x, [(VIDEO, 0, Fr, Hh, W, 0)], Kt, wt, wi, wv)[0, :, 0].reshape(Fr, Hh, W)
    expect = np.zeros((Fr, Hh, W))
    for tau in range(3):
        for a in range(3):
            for e in range(3):
                expect[f0 + 2 - tau, r0 + 1 - a, c0 + 1 - e] = wv[0, 0, tau, a, e]
    assert np.abs(y - expect).max() == 0.0
    assert np.all(y[:f0] == 0.0)


def test_constant_input_interior_sums_and_boundary_partial_sums():
    C, Kt = 2, 4
    rng = np.random.default_rng(3)
    wt, wi, wv = _weights(rng, C, Kt)
    Fr, Hh, W = 4, 4, 5
    x = np.ones((1, Fr * Hh * W, C))
    y = O.mshortconv(x, [(VIDEO, 0, Fr, Hh, W, 0)], Kt, wt, wi, wv)[0].reshape(Fr, Hh, W, C)
    # from frame 2 on, an interior position sees all 27 taps
    assert np.allclose(y[2, 1, 1], wv[0].reshape(C, -1).sum(1), atol=1e-12)
    # frame 0 sees only the current-frame slice (tau = 2); a corner only 4 of its taps
    assert np.allclose(y[0, 0, 0], wv[0, :, 2, 1:, 1:].reshape(C, -1).sum(1), atol=1e-12)
    x = np.ones((1, 10, C))
    y = O.mshortconv(x, [(TEXT, 0, 1, 1, 10, 0)], Kt, wt, wi, wv)[0]
    assert np.allclose(y[0], wt[0, :, Kt - 1], atol=1e-12)
    assert np.allclose(y[5], wt[0].sum(1), atol=1e-12)


def test_image_equals_one_frame_video_with_current_slice():
    """An image is the one-frame case of the visual conv (section 3.4): with causal
    temporal padding only the current-frame slice w[:, 2] of the 3-D kernel acts."""
    C, Kt = 3, 4
    rng = np.random.default_rng(4)
    wt, wi, wv = _weights(rng, C, Kt)
    Hh, W = 6, 7
    x = rng.standard_normal((2, Hh * W, C))
    y_vid = O.mshortconv(x, [(VIDEO, 0, 1, Hh, W, 0)], Kt, wt, wi, wv)
    wi_slice = np.ascontiguousarray(wv[:, :, 2]).astype(np.float32)
    y_img = O.mshortconv(x, [(IMAGE, 0, 1, Hh, W, 0)], Kt, wt, wi_slice, wv)
    assert np.abs(y_vid - y_img).max() <= 1e-12


def test_no_kernel_crosses_a_segment_boundary():
    rng = np.random.default_rng(5)
    segs, T = _segments()
    C = 2
    wt, wi, wv = _weights(rng, C, 4)
    x = rng.standard_normal((1, T, C))
    y = O.mshortconv(x, segs, 4, wt, wi, wv)
    for (m, s, Fr, Hh, W, ws) in segs:
        n = W if m == TEXT else (Hh * W if m == IMAGE else Fr * Hh * W)
        x2 = x.copy()
        x2[:, :s] = rng.standard_normal(x2[:, :s].shape)
        x2[:, s + n:] = rng.standard_normal(x2[:, s + n:].shape)
        y2 = O.mshortconv(x2, segs, 4, wt, wi, wv)
        assert np.array_equal(y2[:, s:s + n], y[:, s:s + n])


def test_l2norm_heads():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((3, 5, 4 * 8))
    x[1, 2, 8:16] = 0.0
    y = O.l2norm_heads(x, 4).reshape(3, 5, 4, 8)
    n = np.linalg.norm(y, axis=-1)
    assert np.allclose(n[n > 0], 1.0, atol=1e-15)
    assert np.all(y[1, 2, 1] == 0.0)
    xr = x.reshape(3, 5, 4, 8)
    cos = (y * xr).sum(-1) / np.maximum(np.linalg.norm(xr, axis=-1), 1e-300)
    assert np.allclose(cos[n > 0], 1.0, atol=1e-14)


def test_rejects_bad_segment_table():
    x = np.zeros((1, 10, 2))
    w = np.zeros((1, 2, 4), dtype=np.float32)
    with pytest.raises(ValueError):
        O.mshortconv(x, [(TEXT, 5, 1, 1, 10, 0)], 4, w)       # runs past T
    with pytest.raises(ValueError):
        O.mshortconv(x, [(IMAGE, 0, 1, 2, 3, 0)], 4, w)       # no image weights
