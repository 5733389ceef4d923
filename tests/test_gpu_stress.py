"""Many calls of the tensor-core scan in a row, at sizes that exercise the split (one to
many chunks per segment, ragged tails, several heads and rows), the gated and fp32 outputs
and packed samples.  Every inter-role wait of the kernel is bounded, so a hand-off that
went wrong would show up as KDA_ERR_TIMEOUT in the device status word rather than a hang;
the test checks that none occurs and that every output is finite, and compares a few
calls with the fp64 oracle on one head."""
import numpy as np
import pytest
import torch

from linear_attention_sequence_mshortconv_b200 import kda
from oracle import oracle as O
from tests.parity import compare, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(B, T, H, seed, strong=False):
    gen = torch.Generator().manual_seed(seed)
    f = dict(generator=gen)
    unit = lambda z: z / torch.linalg.vector_norm(z, dim=-1, keepdim=True)
    lo, hi = (0.3, 3.0) if strong else (0.001, 0.1)
    d = dict(q=unit(torch.randn(B, T, H, 128, **f)), k=unit(torch.randn(B, T, H, 128, **f)),
             v=torch.randn(B, T, H, 128, **f), g=-(lo + (hi - lo) * torch.rand(B, T, H, 128, **f)),
             beta=torch.sigmoid(torch.randn(B, T, H, **f)))
    return {n: x.to(torch.bfloat16) for n, x in d.items()}


def test_many_calls_no_timeout():
    rng = np.random.default_rng(5)
    shapes = [(1, 8192, 4), (1, 4096, 16), (2, 3000, 8), (1, 64 * 150 + 17, 2), (3, 777, 5), (1, 20000, 1),
              (4, 1000, 16), (1, 65, 16), (2, 12345, 3)]
    checked = 0
    for it in range(24):
        B, T, H = shapes[it % len(shapes)]
        strong = it % 5 == 4
        cpu = _inputs(B, T, H, seed=100 + it, strong=strong)
        t = {n: x.to(DEV) for n, x in cpu.items()}
        kind = it % 3
        if kind == 0:
            o, S = kda.forward(t["q"], t["k"], t["v"], t["g"], t["beta"], o_dtype=torch.float32)
        elif kind == 1:
            o, S = kda.forward(t["q"], t["k"], t["v"], t["g"], t["beta"], o_dtype=torch.bfloat16)
        else:
            gate = torch.randn(B, T, H, 128, generator=torch.Generator().manual_seed(it)).to(torch.bfloat16).to(DEV)
            gamma = torch.ones(H, 128, device=DEV)
            o, S = kda.forward_gated(t["q"], t["k"], t["v"], t["g"], t["beta"], gate, gamma, 1e-6)
        torch.cuda.synchronize()
        assert kda.last_device_error() == 0, f"call {it}: device status (B={B}, T={T}, H={H})"
        assert torch.isfinite(o.float()).all() and torch.isfinite(S).all(), f"call {it}: non-finite output"
        if kind == 0 and T * H <= 40000 and checked < 3:
            h = int(rng.integers(H))
            oo, so = O.kda_forward_head(cpu["q"], cpu["k"], cpu["v"], cpu["g"], cpu["beta"], B - 1, h)
            compare(to_np(o)[B - 1, :, h], oo, "bf16", f"call {it} o[b={B - 1},h={h}]")
            compare(to_np(S)[B - 1, h], so, "bf16", f"call {it} S_T[b={B - 1},h={h}]")
            checked += 1
    assert checked >= 1


def test_many_packed_sample_calls_no_timeout():
    rng = np.random.default_rng(6)
    for it in range(8):
        n = int(rng.integers(1, 9))
        lens = [int(x) for x in rng.integers(0, 3000, size=n)]
        cu = [0]
        for L in lens:
            cu.append(cu[-1] + L)
        T = cu[-1]
        if T == 0:
            continue
        cpu = _inputs(1, T, 4, seed=300 + it)
        t = {k: v[0].to(DEV) for k, v in cpu.items()}   # packed axis: [T_total, H, ...]
        o, S = kda.forward_varlen(t["q"], t["k"], t["v"], t["g"], t["beta"], cu, o_dtype=torch.float32)
        torch.cuda.synchronize()
        assert kda.last_device_error() == 0, f"varlen call {it}"
        assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
