"""GPU parity of kda_forward at strong and uneven decay, against the fp64 oracle.

Eq. 14 of the Chimera paper (section 3.3) puts no lower bound on the per-channel forget
gate alpha_t in (0, 1).  On the tensor-core path a chunk whose log-decay range is too
wide for one middle-row reference factorisation takes per-channel references at the
chunk start and end (every factor <= 1) and forms the intra-chunk matrices A and P from
pairwise exponentials instead; these tests put inputs on both sides of that switch, in
the state pass of the segment split as well as in the output pass.
"""
import numpy as np
import pytest
import torch

from linear_attention_sequence_mshortconv_b200 import kda
from oracle import oracle as O
from tests.parity import compare, compare_heads, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(B, T, H, g, seed, S0=False):
    gen = torch.Generator().manual_seed(seed)
    f = dict(generator=gen)
    unit = lambda z: z / torch.linalg.vector_norm(z, dim=-1, keepdim=True)
    d = dict(q=unit(torch.randn(B, T, H, 128, **f)), k=unit(torch.randn(B, T, H, 128, **f)),
             v=torch.randn(B, T, H, 128, **f), g=g, beta=torch.sigmoid(torch.randn(B, T, H, **f)))
    d = {n: x.to(torch.bfloat16) for n, x in d.items()}
    d["S0"] = 0.3 * torch.randn(B, H, 128, 128, **f) if S0 else None
    return d


def _check(d, what, o_dtype=torch.float32):
    t = {n: (x.to(DEV) if x is not None else None) for n, x in d.items()}
    o, ST = kda.forward(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], o_dtype=o_dtype)
    torch.cuda.synchronize()
    assert kda.last_device_error() == 0
    S0 = None if d["S0"] is None else d["S0"].double().numpy()
    o_ref, S_ref = O.kda_forward(d["q"], d["k"], d["v"], d["g"], d["beta"], S0)
    compare_heads(to_np(o), o_ref, to_np(ST), S_ref, "bf16", what=what)


def _uniform(B, T, H, lo, hi, seed):
    gen = torch.Generator().manual_seed(seed)
    return -(lo + (hi - lo) * torch.rand(B, T, H, 128, generator=gen))


@pytest.mark.parametrize("T,S0", [(300, False), (2000, True)])
def test_strong_decay_everywhere(T, S0):
    # g ~ -U(0.3, 3): alpha between 0.05 and 0.74 on every channel; every chunk is too wide
    # for the middle-row reference.  T = 2000 with 2 heads runs the segment split.
    _check(_inputs(1, T, 2, _uniform(1, T, 2, 0.3, 3.0, T), seed=T, S0=S0), f"g~-U(0.3,3) T={T}")


@pytest.mark.parametrize("T", [300, 2000])
def test_one_forgetting_channel_next_to_slow_ones(T):
    # most channels nearly keep their state, a few forget almost completely (alpha = e^-20)
    # on every token, one forgets only on some tokens
    g = _uniform(1, T, 2, 0.001, 0.05, T + 1)
    g[..., 5] = -20.0
    g[:, :, 1, 77] = -20.0
    g[:, ::7, :, 100] = -12.0
    _check(_inputs(1, T, 2, g, seed=T + 2, S0=True), f"mixed channels T={T}")


def test_isolated_near_total_forgetting():
    # single tokens that wipe a channel (alpha = e^-80), otherwise slow decay
    T = 700
    g = _uniform(1, T, 3, 0.001, 0.1, 9)
    g[0, 100, :, :] = -80.0
    g[0, 333, 1, 17:40] = -80.0
    _check(_inputs(1, T, 3, g, seed=10, S0=True), "isolated forgetting")


def test_tiny_config_gate_formula_at_full_width():
    # the tiny workload's alpha = exp(-0.1 softplus(z)) at d = 128 in bf16
    T = 500
    gen = torch.Generator().manual_seed(11)
    g = -0.1 * torch.nn.functional.softplus(torch.randn(1, T, 2, 128, generator=gen))
    _check(_inputs(1, T, 2, g, seed=12), "g = -0.1 softplus(z)")


def test_threshold_region():
    # decay around the switch: some chunks on each side of it
    T = 640
    g = _uniform(1, T, 2, 0.0, 0.6, 13)
    _check(_inputs(1, T, 2, g, seed=14, S0=True), "threshold region")


def test_fp32_inputs_strong_decay():
    # the CUDA-core path (fp32) forms pairwise exponentials directly
    T = 200
    gen = torch.Generator().manual_seed(15)
    f = dict(generator=gen)
    unit = lambda z: z / torch.linalg.vector_norm(z, dim=-1, keepdim=True)
    d = dict(q=unit(torch.randn(1, T, 2, 64, **f)), k=unit(torch.randn(1, T, 2, 64, **f)),
             v=torch.randn(1, T, 2, 64, **f), g=-(0.3 + 2.7 * torch.rand(1, T, 2, 64, **f)),
             beta=torch.sigmoid(torch.randn(1, T, 2, **f)))
    t = {n: x.to(DEV) for n, x in d.items()}
    o, ST = kda.forward(t["q"], t["k"], t["v"], t["g"], t["beta"])
    torch.cuda.synchronize()
    o_ref, S_ref = O.kda_forward(d["q"], d["k"], d["v"], d["g"], d["beta"])
    compare_heads(to_np(o), o_ref, to_np(ST), S_ref, "fp32", what="fp32 strong decay")
