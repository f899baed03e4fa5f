"""Sequence-parallel Lightning prefill: one sequence split into contiguous token segments,
one segment per rank of a torch.distributed group (one process per GPU).

The recurrence S_t = S_{t-1} + kh_t v_t^T is a sum, so a segment's start state is the
initial state plus the state contributions of the segments before it (MiniCPM-SALA
summary page, "Prerequisites / Linear Attention").  Per rank r holding tokens
[p_r, p_r + T_r):
  1. dS_r  = sum over its tokens of kh_t v_t^T, RoPE positions from p_r   (sala_lightning_state)
  2. all ranks' dS gathered                                                (one all-gather)
  3. S0_r  = S_init + sum_{r' < r} dS_r'                                   (sala_state_prefix_sum)
  4. o_r, S_end_r = the ordinary prefill of the segment from S0_r at p_r   (sala_lightning_prefill)
The exchange is D*D*H*B fp32 per rank (2 MiB at H32 D128), once per layer.  Step 1 reads
the segment's k and v once more than a single-device prefill does.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch


def seqpar_prefill(q, k, v, g, S_init, *, rank: int, offsets: Sequence[int], pos0: int,
                   gather_states: Callable, state_fn: Callable, prefix_fn: Callable,
                   prefill_fn: Callable):
    """Steps 1-4 for this rank, with the compute and the collective passed in:
      state_fn(k, v, pos)            -> this segment's state contribution [B,H,D,D]
      gather_states(dS)              -> [world, B,H,D,D], rank order
      prefix_fn(gathered, rank, S0)  -> S0 + sum of gathered[:rank]
      prefill_fn(q, k, v, g, S0, pos)-> (o, S_end)
    `offsets[r]` is the first token of rank r's segment within the sequence."""
    pos = pos0 + int(offsets[rank])
    dS = state_fn(k, v, pos)
    gathered = gather_states(dS)
    S0 = prefix_fn(gathered, rank, S_init)
    return prefill_fn(q, k, v, g, S0, pos)


def lightning_prefill_seqpar(q, k, v, g=None, state=None, q_norm_w=None, k_norm_w=None, *,
                             group=None, chunk=128, pos0=0, rope_base=10000.0, eps=1e-6,
                             out=None, workspace=None):
    """Sequence-parallel Lightning prefill of this rank's segment q, k, v, g [B,T_r,H,D] on
    this rank's GPU.  `state` [B,H,D,D] fp32: the state before the whole sequence (rank 0's
    start; zero when None), the same on every rank.  Returns (out, S_end): the segment's
    outputs and the state after it (on the last rank, the state after the whole sequence)."""
    import torch.distributed as dist

    import sparse_attention_long_lightning_b200 as sala

    rank, world = dist.get_rank(group), dist.get_world_size(group)
    B, T, H, D = q.shape
    lens = torch.zeros(world, dtype=torch.int64, device=q.device)
    dist.all_gather_into_tensor(lens, torch.tensor([T], dtype=torch.int64, device=q.device),
                                group=group)
    offsets = [0] + torch.cumsum(lens, 0).tolist()[:-1]
    need = sala.lightning_prefill_workspace(B, T, H, D, chunk, dtype=q.dtype)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    S_init = (torch.zeros((B, H, D, D), dtype=torch.float32, device=q.device)
              if state is None else state)

    def state_fn(kk, vv, pos):
        return sala.lightning_state(kk, vv, None, k_norm_w, chunk=chunk, pos0=pos,
                                    rope_base=rope_base, eps=eps, workspace=workspace)

    def gather_states(dS):
        gathered = torch.empty((world,) + tuple(dS.shape), dtype=dS.dtype, device=dS.device)
        dist.all_gather_into_tensor(gathered, dS.contiguous(), group=group)
        return gathered

    def prefix_fn(gathered, r, S0):
        start = S0.clone()
        return sala.state_prefix_sum(gathered, r, start, accumulate=True)

    def prefill_fn(qq, kk, vv, gg, S0, pos):
        return sala.lightning_prefill(qq, kk, vv, gg, S0, q_norm_w, k_norm_w, chunk=chunk,
                                      pos0=pos, rope_base=rope_base, eps=eps, out=out,
                                      workspace=workspace)

    return seqpar_prefill(q, k, v, g, S_init, rank=rank, offsets=offsets, pos0=pos0,
                          gather_states=gather_states, state_fn=state_fn, prefix_fn=prefix_fn,
                          prefill_fn=prefill_fn)
