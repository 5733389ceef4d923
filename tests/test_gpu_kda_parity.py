"""GPU parity of kda_forward against the fp64 oracle (through the C ABI binding).

Small problems are compared element by element on every (b, h); the full-size
workloads are compared on sampled heads over their whole length (each head's scan is
independent, so a sampled head is checked exactly, not approximately).
Tolerances are in tests/parity.py.  Parity is measured on the fp32 output (o_dtype =
fp32); a bf16 output is checked to be exactly that fp32 output rounded to nearest even,
since bf16 rounding of o alone can exceed 2% of RMS(o) on heavy-tailed outputs.
"""
import numpy as np
import pytest
import torch

from linear_attention_sequence_mshortconv_b200 import inputs as W
from linear_attention_sequence_mshortconv_b200 import kda
from oracle import oracle as O
from tests.parity import compare, compare_bf16_output, compare_heads, to_np, tol_for

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run_gpu(inp, chunk=0, S0=None, o_dtype=torch.float32):
    t = {k: v.to(DEV) for k, v in inp.items() if isinstance(v, torch.Tensor)}
    S0d = S0.to(DEV) if S0 is not None else None
    o, ST = kda.forward(t["q"], t["k"], t["v"], t["g"], t["beta"], S0d, chunk=chunk,
                        o_dtype=o_dtype)
    torch.cuda.synchronize()
    assert kda.last_device_error() == 0
    return o, ST


def _oracle(inp, S0=None, pairs=None):
    return O.kda_forward(inp["q"].cpu(), inp["k"].cpu(), inp["v"].cpu(), inp["g"].cpu(),
                         inp["beta"].cpu(), None if S0 is None else S0.double().numpy(), pairs=pairs)


def _custom(B, T, H, Dk, Dv, dtype, seed, g_hi=0.1):
    gen = torch.Generator().manual_seed(seed)
    f = dict(generator=gen, dtype=torch.float32)
    unit = lambda z: z / torch.linalg.vector_norm(z, dim=-1, keepdim=True)
    q = unit(torch.randn(B, T, H, Dk, **f))
    k = unit(torch.randn(B, T, H, Dk, **f))
    v = torch.randn(B, T, H, Dv, **f)
    g = -(0.001 + (g_hi - 0.001) * torch.rand(B, T, H, Dk, **f))
    beta = torch.sigmoid(torch.randn(B, T, H, **f))
    return dict(q=q.to(dtype), k=k.to(dtype), v=v.to(dtype), g=g.to(dtype), beta=beta.to(dtype))


def test_tiny_fp32_workload_full():
    w = W.TINY_FP32
    inp = W.make_kda_inputs(w)
    o, ST = _run_gpu(inp, chunk=w.chunk)
    o_ref, S_ref = _oracle(inp)
    compare_heads(to_np(o), o_ref, to_np(ST), S_ref, "fp32", what=w.name)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,T,H,Dk,Dv", [(2, 300, 3, 128, 128), (1, 97, 2, 64, 64),
                                         (1, 130, 2, 32, 128), (1, 65, 1, 128, 32)])
def test_small_shapes_ragged_tail(dtype, B, T, H, Dk, Dv):
    inp = _custom(B, T, H, Dk, Dv, dtype, seed=B * 1000 + T + Dk)
    o, ST = _run_gpu(inp)
    o_ref, S_ref = _oracle(inp)
    compare_heads(to_np(o), o_ref, to_np(ST), S_ref, tol_for(dtype), what=f"{dtype} {B}x{T}x{H}")


@pytest.mark.parametrize("B,T,H", [(2, 150, 80), (1, 1000, 1), (3, 700, 5)])
def test_many_heads_and_segment_splits(B, T, H):
    """Covers one segment per head (B*H >= SM count) and long per-head segment chains."""
    inp = _custom(B, T, H, 128, 128, torch.bfloat16, seed=B * T + H)
    o, ST = _run_gpu(inp)
    pairs = [(b, h) for b in range(B) for h in range(H)][:12]
    o_ref, S_ref = _oracle(inp, pairs=pairs)
    compare_heads(to_np(o), o_ref, to_np(ST), S_ref, "bf16", pairs=pairs, what=f"{B}x{T}x{H}")


@pytest.mark.parametrize("T", [1, 2, 15, 16, 17, 63, 64, 65])
def test_short_and_boundary_lengths(T):
    inp = _custom(1, T, 2, 128, 128, torch.bfloat16, seed=T)
    o, ST = _run_gpu(inp)
    o_ref, S_ref = _oracle(inp)
    compare_heads(to_np(o), o_ref, to_np(ST), S_ref, "bf16", what=f"T={T}")


@pytest.mark.parametrize("chunk", [16, 32, 64, 128])
def test_chunk_size_does_not_change_the_result(chunk):
    inp = _custom(1, 200, 2, 128, 128, torch.bfloat16, seed=5)
    o, ST = _run_gpu(inp, chunk=chunk)
    o_ref, S_ref = _oracle(inp)
    compare_heads(to_np(o), o_ref, to_np(ST), S_ref, "bf16", what=f"chunk={chunk}")


@pytest.mark.parametrize("B,T,H,Dk,Dv,g_hi", [(1, 300, 2, 32, 64, 0.1), (2, 129, 1, 64, 32, 0.1),
                                              (1, 128, 1, 128, 128, 0.1), (1, 257, 1, 128, 32, 3.0)])
def test_chunk_128_fp32(B, T, H, Dk, Dv, g_hi):
    """128-token chunks (key channels taken in blocks of 32): every head width, a chunk
    that is exactly the sequence, ragged tails, an initial state, and strong decay."""
    inp = _custom(B, T, H, Dk, Dv, torch.float32, seed=T + Dk, g_hi=g_hi)
    S0 = torch.randn(B, H, Dk, Dv, generator=torch.Generator().manual_seed(T)) * 0.3
    o, ST = _run_gpu(inp, chunk=128, S0=S0)
    o_ref, S_ref = _oracle(inp, S0=S0)
    compare_heads(to_np(o), o_ref, to_np(ST), S_ref, "fp32", what=f"chunk 128 {B}x{T}x{H} {Dk}x{Dv}")


def test_initial_state_and_split_resume():
    inp = _custom(2, 180, 2, 128, 128, torch.bfloat16, seed=8)
    S0 = torch.randn(2, 2, 128, 128, generator=torch.Generator().manual_seed(1)) * 0.3
    o, ST = _run_gpu(inp, S0=S0)
    o_ref, S_ref = _oracle(inp, S0=S0)
    compare_heads(to_np(o), o_ref, to_np(ST), S_ref, "bf16", what="S0")
    # two calls with S_T -> S0 equal one call
    t0 = 77
    first = {k: v[:, :t0].contiguous() for k, v in inp.items()}
    second = {k: v[:, t0:].contiguous() for k, v in inp.items()}
    o1, S1 = _run_gpu(first, S0=S0)
    o2, S2 = _run_gpu(second, S0=S1.cpu())
    compare_heads(np.concatenate([to_np(o1), to_np(o2)], 1), o_ref, to_np(S2), S_ref, "bf16",
                  what="split")


def test_empty_and_degenerate():
    # T = 0: S_T = S0, o untouched
    z = torch.zeros(1, 0, 2, 64, dtype=torch.bfloat16, device=DEV)
    S0 = torch.randn(1, 2, 64, 64, device=DEV)
    o, ST = kda.forward(z, z, z, z, torch.zeros(1, 0, 2, dtype=torch.bfloat16, device=DEV), S0)
    assert o.shape == (1, 0, 2, 64)
    torch.cuda.synchronize()
    assert torch.equal(ST, S0)
    # beta = 0 and g = 0: the state never changes and o_t = S0^T q_t
    inp = _custom(1, 40, 1, 64, 64, torch.float32, seed=3)
    inp["beta"].zero_()
    inp["g"].zero_()
    S0 = torch.randn(1, 1, 64, 64)
    o, ST = _run_gpu(inp, S0=S0)
    ref = torch.einsum("bthi,bhij->bthj", inp["q"].double(), S0.double())
    compare(to_np(o)[0, :, 0], ref.numpy()[0, :, 0], "fp32", "beta=0,g=0")
    compare(to_np(ST)[0, 0], S0.double().numpy()[0, 0], "fp32", "S_T=S0")


@pytest.mark.parametrize("B,T,H", [(1, 200, 2), (2, 4352, 3)])
def test_bf16_output_is_the_rounded_fp32_output(B, T, H):
    inp = _custom(B, T, H, 128, 128, torch.bfloat16, seed=T)
    o32, S32 = _run_gpu(inp, o_dtype=torch.float32)
    o16, S16 = _run_gpu(inp, o_dtype=torch.bfloat16)
    assert o16.dtype == torch.bfloat16
    assert torch.equal(o16, o32.to(torch.bfloat16))
    assert torch.equal(S16, S32)


def test_heads_and_batches_independent():
    inp = _custom(2, 150, 3, 128, 128, torch.bfloat16, seed=12)
    o, ST = _run_gpu(inp)
    perm_h = [2, 0, 1]
    perm = {k: (v[:, :, perm_h] if v.dim() >= 3 else v).flip(0).contiguous() for k, v in inp.items()}
    o2, ST2 = _run_gpu(perm)
    assert torch.equal(o2, o[:, :, perm_h].flip(0))
    assert torch.equal(ST2, ST[:, perm_h].flip(0))


def test_workspace_is_reused_and_checked():
    inp = _custom(1, 256, 4, 128, 128, torch.bfloat16, seed=2)
    need = kda.workspace_size(1, 256, 4, 128, 128)
    assert need == kda.workspace_size(1, 256, 4, 128, 128, o_dtype=torch.float32)
    t = {k: v.to(DEV) for k, v in inp.items()}
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=DEV)
    o1, S1 = kda.forward(t["q"], t["k"], t["v"], t["g"], t["beta"], workspace=ws)
    o2, S2 = kda.forward(t["q"], t["k"], t["v"], t["g"], t["beta"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    if need > 0:
        small = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
        with pytest.raises(kda.KdaError):
            kda.forward(t["q"], t["k"], t["v"], t["g"], t["beta"], workspace=small)


def _sampled_full_size(w: W.Workload, pairs):
    inp = W.make_kda_inputs(w, device=DEV)
    o, ST = kda.forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], chunk=w.chunk,
                        o_dtype=torch.float32)
    torch.cuda.synchronize()
    assert kda.last_device_error() == 0
    cpu = {k: v.cpu() for k, v in inp.items() if isinstance(v, torch.Tensor)}
    o_np = o[:, :, [h for _, h in pairs]].float().cpu().numpy()
    ST_np = ST.cpu().numpy()
    for idx, (b, h) in enumerate(pairs):
        o_ref, S_ref = O.kda_forward_head(cpu["q"], cpu["k"], cpu["v"], cpu["g"], cpu["beta"], b, h)
        compare(o_np[b, :, idx], o_ref, "bf16", f"{w.name} o[b={b},h={h}]")
        compare(ST_np[b, h], S_ref, "bf16", f"{w.name} S_T[b={b},h={h}]")


def test_image_stream_full_size_sampled_heads():
    _sampled_full_size(W.IMAGE_STREAM, [(0, 0), (3, 15), (1, 7)])


def test_video_clip_full_size_sampled_heads():
    _sampled_full_size(W.VIDEO_CLIP, [(0, 0), (0, 9)])


def test_video_clip_full_size_bf16_output_sampled_heads():
    # the output the benchmark writes: bf16 o (its fp32 form is checked above)
    w = W.VIDEO_CLIP
    inp = W.make_kda_inputs(w, device=DEV)
    o, ST = kda.forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], chunk=w.chunk,
                        o_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert kda.last_device_error() == 0 and o.dtype == torch.bfloat16
    cpu = {k: v.cpu() for k, v in inp.items() if isinstance(v, torch.Tensor)}
    for h in (0, 9):
        o_ref, S_ref = O.kda_forward_head(cpu["q"], cpu["k"], cpu["v"], cpu["g"], cpu["beta"], 0, h)
        compare_bf16_output(to_np(o[0, :, h]), o_ref, f"video clip bf16 o[h={h}]")
        compare(to_np(ST[0, h]), S_ref, "bf16", f"video clip S_T[h={h}]")


def test_long_video_full_size_sampled_head():
    _sampled_full_size(W.LONG_VIDEO, [(0, 5)])


@pytest.mark.parametrize("B,T,H", [(1, 129, 2), (1, 100, 3), (37, 200, 2), (25, 300, 3), (3, 777, 2)])
def test_two_wave_split_boundaries(B, T, H):
    # the uniform-batch split on the tensor-core path: 3 segments (one state-pass segment),
    # 2 segments (no state pass: segment 1 starts from segment 0's end state), W = 2 and
    # W = 1 CTAs per head (74 and 75 heads), and many one-chunk segments with S0 given
    inp = _custom(B, T, H, 128, 128, torch.bfloat16, seed=B * 1000 + T)
    S0 = torch.randn(B, H, 128, 128, generator=torch.Generator().manual_seed(T)) * 0.3
    P, L = kda.forward_plan(B, T, H, 128, 128, torch.bfloat16)
    NC = (T + 63) // 64
    # segments of L chunks (the last may be shorter), or segment 0 the rest, up to 1.04 L
    first = NC - (P - 1) * L
    assert P >= 1 and (P == 1 or (P - 1) * L < NC <= P * L or L < first <= (26 * L + 24) // 25)
    o, ST = _run_gpu(inp, S0=S0)
    o_ref, S_ref = _oracle(inp, S0)
    compare_heads(to_np(o), o_ref, to_np(ST), S_ref, "bf16", what=f"two-wave P={P} L={L}")


def test_forward_is_capturable_in_a_cuda_graph():
    # the two-wave split (device-built work tables, an auxiliary stream joined by events)
    # recorded once in a CUDA graph and replayed: the replay reproduces the eager result
    B, T, H = 1, 3000, 4
    inp = _custom(B, T, H, 128, 128, torch.bfloat16, seed=77)
    t = {k_: v_.to(DEV) for k_, v_ in inp.items()}
    wsz = kda.workspace_size(B, T, H, 128, 128, torch.bfloat16)
    ws = torch.empty(max(wsz, 1), dtype=torch.uint8, device=DEV)
    o = torch.empty(B, T, H, 128, dtype=torch.float32, device=DEV)
    ST = torch.empty(B, H, 128, 128, dtype=torch.float32, device=DEV)
    call = lambda: kda.forward(t["q"], t["k"], t["v"], t["g"], t["beta"], o=o, S_T=ST, workspace=ws,
                               o_dtype=torch.float32)
    call()
    torch.cuda.synchronize()
    o_eager, S_eager = o.clone(), ST.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    o.zero_()
    ST.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert kda.last_device_error() == 0
    assert torch.equal(o, o_eager) and torch.equal(ST, S_eager)
