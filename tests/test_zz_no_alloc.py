"""kda_forward_noalloc against the oracle and against kda_forward.

kda_forward_noalloc exists for callers that cannot allocate device memory during a
call (code inside a framework that owns all device memory through its own allocator,
serving loops on a fixed memory plan).  Its scratch is one array compiled into the
library and shared by every call.  This test makes two calls in a row with different
shapes, the second needing less scratch than the first, so the second runs over the
first call's leftovers laid out for another split.  Each result is checked against the
fp64 oracle on sampled heads at the bf16 parity bound, and must be bit-identical to
kda_forward on the same inputs (same plan, same kernels).  The file is named to be
collected last.
"""
import pytest
import torch

from linear_attention_sequence_mshortconv_b200 import kda
from oracle import oracle as O
from tests.parity import compare, to_np

pytestmark = pytest.mark.gpu


def _inputs(B, T, H, seed):
    gen = torch.Generator().manual_seed(seed)
    unit = lambda z: z / torch.linalg.vector_norm(z, dim=-1, keepdim=True)
    f = dict(generator=gen)
    q = unit(torch.randn(B, T, H, 128, **f))
    k = unit(torch.randn(B, T, H, 128, **f))
    v = torch.randn(B, T, H, 128, **f)
    g = -(0.001 + 0.099 * torch.rand(B, T, H, 128, **f))
    beta = torch.sigmoid(torch.randn(B, T, H, **f))
    S0 = 0.3 * torch.randn(B, H, 128, 128, **f)
    d = lambda t: t.to(torch.bfloat16)
    return d(q), d(k), d(v), d(g), d(beta), S0


def test_noalloc_matches_oracle_and_allocating_entry_point_on_two_calls():
    # B*H = 8 (16 segments of 4 chunks per head on a 148-SM part), then B*H = 16 (8
    # segments of 2 chunks): the tensor-core path keeps the segment maps and start states
    # in the scratch, in a different layout for each call
    shapes = [(1, 4096, 8, 1), (1, 1024, 16, 2)]
    needs = [kda.workspace_size(B, T, H, 128, 128) for B, T, H, _ in shapes]
    assert 0 < needs[1] < needs[0] <= kda.NOALLOC_SCRATCH_BYTES
    cases = [_inputs(B, T, H, seed) for B, T, H, seed in shapes]
    dev = [[t.cuda() for t in c] for c in cases]
    got = []
    for q, k, v, g, beta, S0 in dev:   # the two no-alloc calls back to back
        got.append(kda.forward_noalloc(q, k, v, g, beta, S0, o_dtype=torch.float32))
    torch.cuda.synchronize()
    assert kda.last_device_error() == 0
    for (B, T, H, seed), (q, k, v, g, beta, S0), cpu, (o, S) in zip(shapes, dev, cases, got):
        o_ref, S_ref = kda.forward(q, k, v, g, beta, S0, o_dtype=torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref), f"noalloc o differs from kda_forward (T={T}, H={H})"
        assert torch.equal(S, S_ref), f"noalloc S_T differs from kda_forward (T={T}, H={H})"
        qc, kc, vc, gc, bc, S0c = cpu
        for h in (0, H - 1):
            oo, so = O.kda_forward_head(qc, kc, vc, gc, bc, 0, h, S0_head=S0c[0, h].double().numpy())
            compare(to_np(o)[0, :, h], oo, "bf16", f"noalloc o T={T} h={h}")
            compare(to_np(S)[0, h], so, "bf16", f"noalloc S_T T={T} h={h}")
