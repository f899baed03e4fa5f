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


# ---------------------------------------------------------------------------------------
# Query-range-parallel sparse layer.  One sequence split into contiguous token segments,
# one per rank (as for the sequence-parallel Lightning prefill).  A query row's selection
# and attention read the keys/values of every earlier position, so each rank first
# gathers the whole sequence's k and v (one all-gather each, into its own HBM: no kernel
# reads a peer's memory) and then computes the selection and attention of its own query
# rows only, at their positions in the sequence (sala_sparse_select_rows,
# sala_sparse_attn_rows).  The rows are independent, so the result equals the single-
# device layer row for row; it scales with the number of ranks (not bounded by Hkv like
# the KV-head split), at the cost of every rank holding all of k and v (1 GiB at 1M tokens,
# 2 KV heads, D128, bf16).
# ---------------------------------------------------------------------------------------

def segment_offsets(lens: Sequence[int]):
    """First token of each rank's segment, from the segment lengths in rank order."""
    out, acc = [], 0
    for n in lens:
        if n < 0:
            raise ValueError("segment lengths must be >= 0")
        out.append(acc)
        acc += int(n)
    return out


def gather_token_segments(x, lens: Sequence[int], group=None):
    """Join every rank's contiguous token segment x [B, T_r, ...] (rank order) along the
    token axis into [B, sum(lens), ...] with one all-gather.  Equal segments of a single
    sequence (B = 1) land in place; otherwise the segments are padded to the longest for
    the collective and joined after it."""
    import torch.distributed as dist

    world = len(lens)
    Tm, B, rest = max(lens), x.shape[0], tuple(x.shape[2:])
    if x.shape[1] != lens[dist.get_rank(group)]:
        raise ValueError("x does not hold this rank's segment length")
    if B == 1 and all(n == Tm for n in lens):
        out = torch.empty((1, world * Tm) + rest, dtype=x.dtype, device=x.device)
        dist.all_gather_into_tensor(out.view((world * Tm,) + rest), x[0].contiguous(),
                                    group=group)
        return out
    xp = torch.zeros((B, Tm) + rest, dtype=x.dtype, device=x.device)
    xp[:, :x.shape[1]] = x
    buf = torch.empty((world * B, Tm) + rest, dtype=x.dtype, device=x.device)
    dist.all_gather_into_tensor(buf, xp, group=group)
    buf = buf.view((world, B, Tm) + rest)
    return torch.cat([buf[r, :, :lens[r]] for r in range(world)], dim=1)


def sparse_layer_qrange(q, k, v, g=None, *, rank: int, offsets: Sequence[int],
                        gather_kv: Callable, select_fn: Callable, attn_fn: Callable,
                        gather_fn: Optional[Callable] = None):
    """This rank's share of a sparse layer split over query ranges.  q, g [B,T_r,Hq,D] and
    k, v [B,T_r,Hkv,D] are the rank's token segment, which starts at position
    offsets[rank].  With the compute and the collectives passed in:
      K, V = gather_kv(k, v)            the whole sequence's keys / values [B,T,Hkv,D]
      idx  = select_fn(q, K, p)         [B,Hkv,T_r,n_sel], q's rows at positions p ..
      o    = attn_fn(q, K, V, idx, g, p) [B,T_r,Hq,D]
    returns o, or the whole [B,T,Hq,D] when `gather_fn(o) -> [B,T,Hq,D]` is given."""
    p = int(offsets[rank])
    K, V = gather_kv(k, v)
    if K.shape[1] < p + q.shape[1]:
        raise ValueError("the gathered keys do not reach this rank's rows")
    idx = select_fn(q, K, p)
    o = attn_fn(q, K, V, idx, g, p)
    return o if gather_fn is None else gather_fn(o)


def sparse_layer_query_parallel(q, k, v, g=None, *, group=None, topk=64, n_init=1, n_local=2,
                                block=64, score="group_sum", gather=True):
    """Query-range-parallel sparse layer on this rank's GPU (one process per GPU, NCCL).
    q, g [B,T_r,Hq,D] and k, v [B,T_r,Hkv,D]: this rank's contiguous token segment of the
    sequence (rank order; lengths may differ).  k and v are all-gathered into this GPU's
    memory, then libsala selects and attends for the rank's rows at their positions.
    Returns the rank's output rows, or with gather=True the whole sequence's output."""
    import torch.distributed as dist

    import sparse_attention_long_lightning_b200 as sala

    rank, world = dist.get_rank(group), dist.get_world_size(group)
    lens_t = torch.zeros(world, dtype=torch.int64, device=q.device)
    dist.all_gather_into_tensor(lens_t, torch.tensor([q.shape[1]], dtype=torch.int64,
                                                     device=q.device), group=group)
    lens = [int(n) for n in lens_t.tolist()]
    offsets = segment_offsets(lens)

    def gather_kv(kk, vv):
        return gather_token_segments(kk, lens, group), gather_token_segments(vv, lens, group)

    def select_fn(qq, K, p):
        return sala.sparse_select(qq, K, topk=topk, n_init=n_init, n_local=n_local, block=block,
                                  score=score, q_pos0=p)

    def attn_fn(qq, K, V, idx, gg, p):
        return sala.sparse_attn(qq, K, V, idx, gg, block=block, q_pos0=p)

    def gather_fn(o):
        return gather_token_segments(o, lens, group)

    return sparse_layer_qrange(q, k, v, g, rank=rank, offsets=offsets, gather_kv=gather_kv,
                               select_fn=select_fn, attn_fn=attn_fn,
                               gather_fn=gather_fn if gather else None)
