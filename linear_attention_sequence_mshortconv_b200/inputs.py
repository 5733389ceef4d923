"""Seeded synthetic workloads for the KDA scan and mShortConv.

This module only draws random numbers in the shapes and distributions of the
benchmark workloads; it holds none of the method's arithmetic, so both the CUDA path
and the CPU oracle can be fed from it.  Values are drawn in fp32 with a seeded
``torch.Generator`` in the fixed order q, k, v, g, beta (then x, w for the fused
workload) and rounded once to the run dtype; every consumer sees the same rounded
values.

Stream layouts follow the single-stream packing of the Chimera paper (section 3.2,
Eq. 2: text tokens first, then visual tokens) and the time-first raster order of
section 3.3, Eq. 12.  A segment is (modality, start, F, Hgt, Wid, weight_set) with
modality 0 = text (F = Hgt = 1, Wid = length), 1 = image (F = 1), 2 = video.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Tuple

import torch

TEXT, IMAGE, VIDEO = 0, 1, 2

Segment = Tuple[int, int, int, int, int, int]


def stream_segments(text: int, visual: List[Tuple[int, int, int, int]]) -> List[Segment]:
    """Text prefix followed by visual blocks given as (modality, F, Hgt, Wid)."""
    segs: List[Segment] = []
    pos = 0
    if text:
        segs.append((TEXT, 0, 1, 1, text, 0))
        pos = text
    for (m, F, Hh, W) in visual:
        segs.append((m, pos, F, Hh, W, 0))
        pos += F * Hh * W
    return segs


def stream_length(segs: List[Segment]) -> int:
    end = 0
    for (m, s, F, Hh, W, _) in segs:
        end = max(end, s + (W if m == TEXT else (Hh * W if m == IMAGE else F * Hh * W)))
    return end


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    D: int
    chunk: int
    dtype: torch.dtype
    seed: int
    segments: Tuple[Segment, ...]
    g_dist: str            # "softplus01": g = -0.1*softplus(N(0,1)); "uniform": g ~ -U(g_lo, g_hi)
    g_lo: float = 0.0
    g_hi: float = 0.0
    beta_dist: str = "sigmoid"   # "uniform": U(0,1); "sigmoid": sigmoid(N(0,1))
    fused: bool = False
    Kt: int = 4
    T_override: Optional[int] = None

    @property
    def T(self) -> int:
        return self.T_override if self.T_override is not None else stream_length(list(self.segments))

    @property
    def tokens(self) -> int:
        return self.B * self.T

    def resized(self, *, B=None, H=None, T=None, name=None) -> "Workload":
        """Same distributions on a smaller problem (segments truncated to the new T)."""
        kw = {}
        if B is not None:
            kw["B"] = B
        if H is not None:
            kw["H"] = H
        if T is not None:
            kw["T_override"] = T
            kw["segments"] = tuple(_truncate(list(self.segments), T))
        kw["name"] = name or (self.name + "_resized")
        return dataclasses.replace(self, **kw)


def _truncate(segs: List[Segment], T: int) -> List[Segment]:
    """Keep the segments that fit in [0, T); the last one is cut to whole rows / frames
    and any remainder is covered by a trailing text run, so the table covers [0, T)."""
    out: List[Segment] = []
    for (m, s, F, Hh, W, ws) in segs:
        if s >= T:
            break
        room = T - s
        if m == TEXT:
            out.append((m, s, 1, 1, min(W, room), ws))
        elif m == IMAGE:
            rows = min(Hh, room // W)
            if rows > 0:
                out.append((m, s, 1, rows, W, ws))
        else:
            frames = min(F, room // (Hh * W))
            if frames > 0:
                out.append((m, s, frames, Hh, W, ws))
    covered = stream_length(out)
    if covered < T:
        out.append((TEXT, covered, 1, 1, T - covered, 0))
    return out


# The five benchmark workloads.  Names say what they are.
TINY_FP32 = Workload("tiny_fp32_B1_H2_T64_d32", B=1, H=2, D=32, chunk=16, dtype=torch.float32,
                     seed=0, segments=((TEXT, 0, 1, 1, 64, 0),), g_dist="softplus01",
                     beta_dist="uniform")
IMAGE_STREAM = Workload("image_stream_B4_H16_T4352_d128", B=4, H=16, D=128, chunk=64,
                        dtype=torch.bfloat16, seed=1,
                        segments=tuple(stream_segments(256, [(IMAGE, 1, 64, 64)])),
                        g_dist="uniform", g_lo=0.001, g_hi=0.1)
VIDEO_CLIP = Workload("video_clip_B1_H16_T32768_d128", B=1, H=16, D=128, chunk=64,
                      dtype=torch.bfloat16, seed=2,
                      segments=tuple(stream_segments(512, [(VIDEO, 21, 32, 48)])),
                      g_dist="uniform", g_lo=0.001, g_hi=0.1)
FUSED_MIXED = Workload("fused_conv_kda_B1_H16_T36864_d128", B=1, H=16, D=128, chunk=64,
                       dtype=torch.bfloat16, seed=3,
                       segments=tuple(stream_segments(512, [(IMAGE, 1, 64, 64), (VIDEO, 21, 32, 48)])),
                       g_dist="uniform", g_lo=0.001, g_hi=0.1, fused=True, Kt=4)
LONG_VIDEO = Workload("long_video_B1_H16_T258560_d128", B=1, H=16, D=128, chunk=64,
                      dtype=torch.bfloat16, seed=4,
                      segments=tuple(stream_segments(512, [(VIDEO, 126, 32, 64)])),
                      g_dist="uniform", g_lo=1e-4, g_hi=0.05)

WORKLOADS = [TINY_FP32, IMAGE_STREAM, VIDEO_CLIP, FUSED_MIXED, LONG_VIDEO]
BY_NAME = {w.name: w for w in WORKLOADS}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _unit_rows(z: torch.Tensor) -> torch.Tensor:
    # The workloads specify L2-normalised Gaussian q and k per (token, head); this is
    # part of the input recipe, not of the scan.
    n = torch.linalg.vector_norm(z, dim=-1, keepdim=True)
    return z / n


def make_kda_inputs(w: Workload, device="cpu"):
    """q, k, g: [B,T,H,D]; v: [B,T,H,D]; beta: [B,T,H]; all in w.dtype; S0 = None."""
    B, T, H, D = w.B, w.T, w.H, w.D
    gen = _gen(w.seed, device)
    f32 = dict(device=device, dtype=torch.float32, generator=gen)
    q = _unit_rows(torch.randn(B, T, H, D, **f32))
    k = _unit_rows(torch.randn(B, T, H, D, **f32))
    v = torch.randn(B, T, H, D, **f32)
    g = _draw_g(w, (B, T, H, D), f32)
    beta = _draw_beta(w, (B, T, H), f32)
    dt = w.dtype
    return dict(q=q.to(dt), k=k.to(dt), v=v.to(dt), g=g.to(dt), beta=beta.to(dt), S0=None)


def _draw_g(w: Workload, shape, f32):
    if w.g_dist == "softplus01":
        return -0.1 * torch.nn.functional.softplus(torch.randn(*shape, **f32))
    u = torch.rand(*shape, **f32)
    return -(w.g_lo + (w.g_hi - w.g_lo) * u)


def _draw_beta(w: Workload, shape, f32):
    if w.beta_dist == "uniform":
        return torch.rand(*shape, **f32)
    return torch.sigmoid(torch.randn(*shape, **f32))


def make_fused_inputs(w: Workload, device="cpu"):
    """x_q, x_k, x_v: [B,T,H*D] in w.dtype; conv weights fp32 per tensor as
    (w_text [1,C,Kt], w_image [1,C,3,3], w_video [1,C,3,3,3]) with N(0, 1/fan_in);
    g [B,T,H,D], beta [B,T,H] with the workload's distributions."""
    B, T, H, D = w.B, w.T, w.H, w.D
    C = H * D
    gen = _gen(w.seed, device)
    f32 = dict(device=device, dtype=torch.float32, generator=gen)
    xs = [torch.randn(B, T, C, **f32).to(w.dtype) for _ in range(3)]
    g = _draw_g(w, (B, T, H, D), f32).to(w.dtype)
    beta = _draw_beta(w, (B, T, H), f32).to(w.dtype)
    weights = []
    for _ in range(3):
        wt = torch.randn(1, C, w.Kt, **f32) / (w.Kt ** 0.5)
        wi = torch.randn(1, C, 3, 3, **f32) / 3.0
        wv = torch.randn(1, C, 3, 3, 3, **f32) / (27 ** 0.5)
        weights.append((wt.contiguous(), wi.contiguous(), wv.contiguous()))
    return dict(xq=xs[0], xk=xs[1], xv=xs[2], wq=weights[0], wk=weights[1], wv=weights[2],
                g=g, beta=beta, segments=list(w.segments))
