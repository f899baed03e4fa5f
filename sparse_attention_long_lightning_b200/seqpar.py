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


# ---------------------------------------------------------------------------------------
# KV-head-parallel sparse layer.  Block selection and block-sparse attention of KV head
# hk touch only hk's keys/values and the query heads of its group (the GQA group shares
# the selection), so ranks that each own a contiguous range of KV heads (with their
# query groups) need no exchange; the only collective is the optional all-gather of the
# outputs along the head axis.  It scales to at most Hkv ranks (2 for 32q/2kv).
# ---------------------------------------------------------------------------------------

def kvhead_range(Hkv: int, rank: int, world: int):
    """KV heads [lo, hi) owned by `rank` of `world` (contiguous, sizes differ by <= 1)."""
    if not 0 <= rank < world or world > Hkv:
        raise ValueError("need 0 <= rank < world <= Hkv")
    return rank * Hkv // world, (rank + 1) * Hkv // world


def sparse_layer_headpar(q, k, v, g=None, *, rank: int, world: int, select_fn: Callable,
                         attn_fn: Callable, gather_fn: Optional[Callable] = None):
    """This rank's share of a sparse layer: q, g [B,T,Hq,D] and k, v [B,T,Hkv,D] hold all
    heads (or views of them); the rank computes
      idx = select_fn(q_r, k_r), o_r = attn_fn(q_r, k_r, v_r, idx, g_r)
    on its KV heads and their query groups (views, no copies) and returns o_r, or the
    full [B,T,Hq,D] output when `gather_fn(o_r) -> list of every rank's o in rank order`
    is given."""
    Hq, Hkv = q.shape[2], k.shape[2]
    grp = Hq // Hkv
    lo, hi = kvhead_range(Hkv, rank, world)
    q_r, g_r = q[:, :, lo * grp:hi * grp], (None if g is None else g[:, :, lo * grp:hi * grp])
    k_r, v_r = k[:, :, lo:hi], v[:, :, lo:hi]
    idx = select_fn(q_r, k_r)
    o_r = attn_fn(q_r, k_r, v_r, idx, g_r)
    if gather_fn is None:
        return o_r
    return torch.cat(list(gather_fn(o_r)), dim=2)


def sparse_layer_kvhead_parallel(q, k, v, g=None, *, group=None, topk=64, n_init=1, n_local=2,
                                 block=64, gather=True):
    """KV-head-parallel sparse layer on this rank's GPU (one process per GPU, NCCL):
    libsala selection and attention on the rank's KV heads; with gather=True the outputs
    of all ranks are all-gathered (every rank's share has the same shape when Hkv is a
    multiple of the world size)."""
    import torch.distributed as dist

    import sparse_attention_long_lightning_b200 as sala

    rank, world = dist.get_rank(group), dist.get_world_size(group)
    if k.shape[2] % world:
        raise ValueError("Hkv must be a multiple of the world size")

    def select_fn(qq, kk):
        return sala.sparse_select(qq, kk, topk=topk, n_init=n_init, n_local=n_local, block=block)

    def attn_fn(qq, kk, vv, idx, gg):
        return sala.sparse_attn(qq, kk, vv, idx, gg, block=block)

    def gather_fn(o_r):
        parts = [torch.empty_like(o_r) for _ in range(world)]
        dist.all_gather(parts, o_r.contiguous(), group=group)
        return parts

    return sparse_layer_headpar(q, k, v, g, rank=rank, world=world, select_fn=select_fn,
                                attn_fn=attn_fn, gather_fn=gather_fn if gather else None)
