"""Sequence-parallel KDA forward over torch.distributed: every rank of a process group
holds one time shard of the same B rows (rank r holds the r-th consecutive run of
tokens) and the ranks together compute what one kda_forward over the whole rows would.

Eq. 14 of the Chimera paper (section 3.3) is affine in the state, so a shard maps its
entry state to S_out = M S_in + N.  The steps, all but the exchange in libkda:
  1. kda_sp_transition: this shard's [N | M] (one state pass of the scan),
  2. one all-gather of every rank's [N | M] (B*H*2*D*D fp32: 2 MiB at H = 16, D = 128),
  3. kda_sp_prefix: the entry state of this shard, shards 0..r-1 folded over S0,
  4. kda_sp_output: this shard's output from that state (one output pass).
The exchange is the only collective, and it carries no token data.

``ops`` holds the three local steps; the default is the CUDA library.  A test can put
any implementation with the same contract there to check the orchestration on CPU
ranks (the gloo backend).
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

from . import kda


class CudaShardOps:
    """The local steps on the CUDA library (the product path)."""

    def workspace(self, q, chunk):
        return kda.sp_workspace(q, chunk)

    def transition(self, q, k, v, g, beta, ws, chunk):
        return kda.sp_transition(q, k, v, g, beta, ws, chunk=chunk)

    def prefix(self, MN_all, r, S0):
        return kda.sp_prefix(MN_all, r, S0)

    def output(self, q, k, v, g, beta, S_in, ws, chunk, o_dtype):
        return kda.sp_output(q, k, v, g, beta, S_in, ws, chunk=chunk, o_dtype=o_dtype)


def _all_gather(MN: torch.Tensor, group) -> torch.Tensor:
    R = dist.get_world_size(group)
    if dist.get_backend(group) == "nccl":
        out = torch.empty((R,) + tuple(MN.shape), dtype=MN.dtype, device=MN.device)
        dist.all_gather_into_tensor(out, MN.contiguous(), group=group)
        return out
    parts = [torch.empty_like(MN) for _ in range(R)]
    dist.all_gather(parts, MN.contiguous(), group=group)
    return torch.stack(parts)


def forward(q, k, v, g, beta, S0: Optional[torch.Tensor] = None, *, group=None, chunk: int = 0,
            o_dtype=None, broadcast_state: bool = False, ops=None):
    """This rank's shard of a sequence-parallel KDA forward.

    q, k, g, v: [B, T_r, H, D] and beta: [B, T_r, H] -- this rank's tokens of the rows
    (shards may differ in length); S0: [B, H, D, D] fp32, the rows' initial state, the
    same on every rank (None = zeros).  Returns (o [B, T_r, H, D], S_T): S_T is this
    shard's final state, which on the last rank is the rows' final state; with
    ``broadcast_state`` every rank receives the last rank's.
    """
    ops = ops or CudaShardOps()
    r = dist.get_rank(group)
    R = dist.get_world_size(group)
    ws = ops.workspace(q, chunk)
    MN = ops.transition(q, k, v, g, beta, ws, chunk)
    MN_all = _all_gather(MN, group)
    S_in = ops.prefix(MN_all, r, S0)
    o, S_T = ops.output(q, k, v, g, beta, S_in, ws, chunk, o_dtype)
    if broadcast_state:
        src = dist.get_global_rank(group, R - 1) if group is not None else R - 1
        dist.broadcast(S_T, src=src, group=group)
    return o, S_T
