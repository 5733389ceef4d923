"""The host side of the sequence-parallel forward on CPU ranks (gloo, world sizes 2 and 3).

sequence_parallel.forward is run with its local steps supplied by the fp64 oracle
(the shard's [N | M] from two oracle scans, the prefix fold in fp64, the shard's scan
from its entry state), so what is checked is the orchestration itself: the all-gather
in rank order, the entry state each rank derives from the others' maps, uneven shard
lengths, and the broadcast of the final state.  The ranks' outputs, concatenated, must
equal the oracle's scan of the whole rows.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUTS = [0, 17, 40]
B, H, D = 2, 2, 8


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rows(seed=21, T=None):
    gen = torch.Generator().manual_seed(seed)
    f = dict(generator=gen, dtype=torch.float64)
    T = T or CUTS[-1]
    unit = lambda z: z / torch.linalg.vector_norm(z, dim=-1, keepdim=True)
    q, k = unit(torch.randn(B, T, H, D, **f)), unit(torch.randn(B, T, H, D, **f))
    v = torch.randn(B, T, H, D, **f)
    g = -(0.001 + 0.099 * torch.rand(B, T, H, D, **f))
    beta = torch.sigmoid(torch.randn(B, T, H, **f))
    S0 = torch.randn(B, H, D, D, **f) * 0.3
    return dict(q=q, k=k, v=v, g=g, beta=beta), S0


class OracleShardOps:
    """The three local steps on the fp64 oracle (test stand-in for the CUDA library)."""

    def __init__(self, O):
        self.O = O

    def workspace(self, q, chunk):
        return None

    def transition(self, q, k, v, g, beta, ws, chunk):
        Bq, T, Hq, Dq = q.shape
        _, N = self.O.kda_forward(q, k, v, g, beta, want_o=False)
        eye = np.broadcast_to(np.eye(Dq), (Bq, Hq, Dq, Dq)).copy()
        _, M = self.O.kda_forward(q, k, torch.zeros_like(v), g, beta, eye, want_o=False)
        return torch.from_numpy(np.stack([N, M], axis=2))

    def prefix(self, MN_all, r, S0):
        S = S0.clone() if S0 is not None else torch.zeros(MN_all.shape[1:3] + MN_all.shape[-2:], dtype=torch.float64)
        for j in range(r):
            S = MN_all[j, :, :, 1] @ S + MN_all[j, :, :, 0]
        return S

    def output(self, q, k, v, g, beta, S_in, ws, chunk, o_dtype):
        o, ST = self.O.kda_forward(q, k, v, g, beta, S_in.numpy())
        return torch.from_numpy(o), torch.from_numpy(ST)


def _worker(rank, port, out, cuts=None):
    cuts = cuts or CUTS
    ws_ = len(cuts) - 1
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws_))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from linear_attention_sequence_mshortconv_b200 import sequence_parallel as sp
    from oracle import oracle as O
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=ws_, timeout=timedelta(seconds=60))
    try:
        inp, S0 = _rows(T=cuts[-1])
        a, b = cuts[rank], cuts[rank + 1]
        shard = {n: x[:, a:b].contiguous() for n, x in inp.items()}
        o, ST = sp.forward(shard["q"], shard["k"], shard["v"], shard["g"], shard["beta"], S0,
                           broadcast_state=True, ops=OracleShardOps(O))
        out.put((rank, o.numpy(), ST.numpy()))
    finally:
        dist.destroy_process_group()


def test_sequence_parallel_orchestration_gloo():
    sys.path.insert(0, ROOT)
    from oracle import oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp, S0 = _rows()
    o_ref, S_ref = O.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0.numpy())
    o = np.concatenate([res[0][1], res[1][1]], axis=1)
    scale = np.abs(o_ref).max()
    assert np.abs(o - o_ref).max() <= 1e-12 * scale
    for r in range(2):   # broadcast_state: every rank holds the rows' final state
        assert np.abs(res[r][2] - S_ref).max() <= 1e-12 * np.abs(S_ref).max()


def test_sequence_parallel_three_ranks_with_an_empty_shard():
    sys.path.insert(0, ROOT)
    from oracle import oracle as O
    cuts = [0, 11, 11, 30]   # rank 1 holds no token: its map is the identity
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q, cuts)) for r in range(3)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp, S0 = _rows(T=cuts[-1])
    o_ref, S_ref = O.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0.numpy())
    o = np.concatenate([r[1] for r in res], axis=1)
    assert np.abs(o - o_ref).max() <= 1e-12 * np.abs(o_ref).max()
    for r in range(3):
        assert np.abs(res[r][2] - S_ref).max() <= 1e-12 * np.abs(S_ref).max()
