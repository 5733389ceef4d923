"""GPU parity of the sequence-parallel calls (kda_sp_transition, kda_sp_prefix,
kda_sp_output) against the fp64 oracle, through the C ABI binding.

The ranks of a sequence-parallel run are emulated one after another in this process
(every kernel runs to completion before the next shard's starts; nothing waits on
another launch): the shards' outputs, concatenated, must match the oracle's scan of the
whole rows, and the last shard's S_T the rows' final state.  Shard lengths mix ragged
tails, an exact chunk, a shard long enough to be split into several segments on the
tensor-core route, and an empty shard.  Each shard's [N | M] is also checked on its own
against the oracle: N is the state reached from zero, M the state reached from S0 = I
with v = 0 (the affine map of Eq. 14 evaluated at two points).
"""
import numpy as np
import pytest
import torch

from linear_attention_sequence_mshortconv_b200 import kda
from oracle import oracle as O
from tests.parity import compare, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _rows(B, T, H, D, dtype, seed, g_lo=0.001, g_hi=0.1):
    gen = torch.Generator().manual_seed(seed)
    f = dict(generator=gen, dtype=torch.float32)
    unit = lambda z: z / torch.linalg.vector_norm(z, dim=-1, keepdim=True)
    q, k = unit(torch.randn(B, T, H, D, **f)), unit(torch.randn(B, T, H, D, **f))
    v = torch.randn(B, T, H, D, **f)
    g = -(g_lo + (g_hi - g_lo) * torch.rand(B, T, H, D, **f))
    beta = torch.sigmoid(torch.randn(B, T, H, **f))
    return {n: t.to(dtype) for n, t in dict(q=q, k=k, v=v, g=g, beta=beta).items()}


def _shard(inp, a, b):
    return {n: x[:, a:b].contiguous() for n, x in inp.items()}


def _run_shards(inp, cuts, S0, chunk=0, o_dtype=torch.float32):
    """Emulated ranks: transition of every shard, then prefix + output of every shard."""
    shards = [{n: x.to(DEV) for n, x in _shard(inp, a, b).items()} for a, b in zip(cuts[:-1], cuts[1:])]
    wss, MNs = [], []
    for s in shards:
        ws = kda.sp_workspace(s["q"], chunk)
        wss.append(ws)
        MNs.append(kda.sp_transition(s["q"], s["k"], s["v"], s["g"], s["beta"], ws, chunk=chunk))
    MN_all = torch.stack(MNs)
    S0d = None if S0 is None else S0.to(DEV)
    os_, STs = [], []
    for r, s in enumerate(shards):
        S_in = kda.sp_prefix(MN_all, r, S0d)
        o, ST = kda.sp_output(s["q"], s["k"], s["v"], s["g"], s["beta"], S_in, wss[r], chunk=chunk,
                              o_dtype=o_dtype)
        os_.append(o)
        STs.append(ST)
    torch.cuda.synchronize()
    assert kda.last_device_error() == 0
    return torch.cat(os_, dim=1), STs[-1], MN_all


def _check_rows(inp, cuts, S0, kind, chunk=0, o_dtype=torch.float32):
    o, ST, MN_all = _run_shards(inp, cuts, S0, chunk, o_dtype)
    o_ref, S_ref = O.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                 None if S0 is None else S0.double().numpy())
    og, Sg = to_np(o), to_np(ST)
    B, T, H, _ = o_ref.shape
    for b in range(B):
        for h in range(H):
            compare(og[b, :, h], o_ref[b, :, h], kind, f"o b={b} h={h}")
            compare(Sg[b, h], S_ref[b, h], kind, f"S_T b={b} h={h}")
    return MN_all


def _check_maps(inp, MN, kind):
    """MN [B,H,2,D,D] of one shard against the oracle at S = 0 and at S = I, v = 0."""
    B, T, H, D = inp["q"].shape
    _, N_ref = O.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], want_o=False)
    eye = np.broadcast_to(np.eye(D), (B, H, D, D)).copy()
    _, M_ref = O.kda_forward(inp["q"], inp["k"], torch.zeros_like(inp["v"]), inp["g"], inp["beta"], eye,
                             want_o=False)
    m = to_np(MN)
    for b in range(B):
        for h in range(H):
            compare(m[b, h, 0], N_ref[b, h], kind, f"N b={b} h={h}")
            compare(m[b, h, 1], M_ref[b, h], kind, f"M b={b} h={h}")


def test_sp_tensor_core_route_bf16():
    # B*H = 6 heads: a 1000-token shard has 16 chunks and is cut into 16 segments
    B, H, D = 2, 3, 128
    cuts = [0, 300, 364, 364, 1364, 1369, 1500]
    inp = _rows(B, cuts[-1], H, D, torch.bfloat16, seed=11)
    S0 = torch.randn(B, H, D, D, generator=torch.Generator().manual_seed(12)) * 0.3
    _check_rows(inp, cuts, S0, "bf16")


def test_sp_bf16_output_and_zero_initial_state():
    B, H, D = 1, 4, 128
    cuts = [0, 640, 1283, 2000]
    inp = _rows(B, cuts[-1], H, D, torch.bfloat16, seed=13)
    _check_rows(inp, cuts, None, "bf16", o_dtype=torch.bfloat16)


def test_sp_shard_maps_bf16():
    # slow decay, so that M stays well inside the range of the fp16 MMA operands
    B, H, D = 1, 2, 128
    inp = _rows(B, 256, H, D, torch.bfloat16, seed=14, g_hi=0.02)
    s = {n: x.to(DEV) for n, x in inp.items()}
    ws = kda.sp_workspace(s["q"])
    MN = kda.sp_transition(s["q"], s["k"], s["v"], s["g"], s["beta"], ws)
    torch.cuda.synchronize()
    _check_maps(inp, MN, "bf16")


@pytest.mark.parametrize("chunk", [16, 128])
def test_sp_cuda_core_route_fp32(chunk):
    B, H, D = 1, 2, 32
    cuts = [0, 50, 66, 143] if chunk == 16 else [0, 130, 140, 400]
    inp = _rows(B, cuts[-1], H, D, torch.float32, seed=15)
    S0 = torch.randn(B, H, D, D, generator=torch.Generator().manual_seed(16)) * 0.3
    MN_all = _check_rows(inp, cuts, S0, "fp32", chunk=chunk)
    _check_maps(_shard(inp, 0, cuts[1]), MN_all[0], "fp32")


def test_sp_prefix_fold_against_float64():
    # the fold of random maps (not produced by a scan) against the same fold in fp64
    R, B, H, D = 4, 1, 2, 64
    gen = torch.Generator().manual_seed(17)
    MN_all = torch.randn(R, B, H, 2, D, D, generator=gen) * 0.1
    S0 = torch.randn(B, H, D, D, generator=gen)
    d_all, d_S0 = MN_all.to(DEV), S0.to(DEV)
    for r in range(R):
        got = to_np(kda.sp_prefix(d_all, r, d_S0))
        S = S0.double()
        for j in range(r):
            S = MN_all[j, :, :, 1].double() @ S + MN_all[j, :, :, 0].double()
        ref = S.numpy()
        for h in range(H):
            compare(got[0, h], ref[0, h], "fp32", f"prefix r={r} h={h}")


def test_sp_empty_shard_is_identity_map():
    B, H, D = 1, 2, 128
    z = torch.empty(B, 0, H, D, dtype=torch.bfloat16, device=DEV)
    MN = kda.sp_transition(z, z, z, z, torch.empty(B, 0, H, dtype=torch.bfloat16, device=DEV), None)
    torch.cuda.synchronize()
    m = to_np(MN)
    assert np.all(m[:, :, 0] == 0.0)
    assert np.all(m[:, :, 1] == np.eye(D))
