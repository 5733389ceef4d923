"""kda_forward_noalloc against kda_forward.

kda_forward_noalloc exists for callers that cannot allocate device memory during a
call (code inside a framework that owns all device memory through its own allocator,
serving loops on a fixed memory plan).  Its scratch is one array compiled into the
library and shared by every call, so this test makes two calls in a row on different
inputs and checks each against the allocating entry point on the same inputs, with the
parity tolerance the other GPU tests use.  The file is named to be collected last.
"""
import pytest
import torch

from linear_attention_sequence_mshortconv_b200 import kda
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
    d = lambda t: t.to(torch.bfloat16).cuda()
    return d(q), d(k), d(v), d(g), d(beta), S0.cuda()


def test_noalloc_matches_allocating_entry_point_on_two_calls():
    # B*H = 4 on a 148-SM part: the tensor-core path cuts each head into segments and
    # uses its scratch for the segment maps and start states.
    B, T, H = 1, 2048, 4
    need = kda.workspace_size(B, T, H, 128, 128)
    assert 0 < need <= kda.NOALLOC_SCRATCH_BYTES
    for seed in (1, 2):
        q, k, v, g, beta, S0 = _inputs(B, T, H, seed)
        o_ref, S_ref = kda.forward(q, k, v, g, beta, S0, o_dtype=torch.float32)
        o, S = kda.forward_noalloc(q, k, v, g, beta, S0, o_dtype=torch.float32)
        torch.cuda.synchronize()
        assert kda.last_device_error() == 0
        for h in range(H):
            compare(to_np(o)[0, :, h], to_np(o_ref)[0, :, h], "bf16", f"noalloc o h={h} seed={seed}")
            compare(to_np(S)[0, h], to_np(S_ref)[0, h], "bf16", f"noalloc S_T h={h} seed={seed}")
