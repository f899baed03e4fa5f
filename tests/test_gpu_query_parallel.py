"""GPU parity: selection and attention over a window of query rows (sala_sparse_select_rows,
sala_sparse_attn_rows) and the query-range-parallel sparse layer built on them.

A window's rows are positions q_pos0 .. q_pos0 + Tq - 1 of the sequence whose k and v
(all Tk positions) are given whole, so each window must reproduce the same rows of the
whole-sequence calls bit for bit (rows are computed independently and, with the same v,
the attention's per-(sequence, KV head) v scale is the same); one window is also checked
against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_long_lightning_b200 import inputs
from tests._parity import TOL_BF16, check_index_sets, rel_err

pytestmark = pytest.mark.gpu

sala = pytest.importorskip("sparse_attention_long_lightning_b200")
DEV = "cuda"


def _np(t):
    return t.detach().double().cpu().numpy()


def _windows_match_whole(s, cuts, *, topk=64, score="group_sum", n_local=2):
    q, k, v, g = s.q, s.k, s.v, s.g
    idx_w = sala.sparse_select(q, k, topk=topk, n_local=n_local, score=score)
    o_w = sala.sparse_attn(q, k, v, idx_w, g)
    for a, b in zip(cuts, cuts[1:]):
        idx = sala.sparse_select(q[:, a:b], k, topk=topk, n_local=n_local, score=score,
                                 q_pos0=a)
        assert torch.equal(idx, idx_w[:, :, a:b]), (a, b)
        o = sala.sparse_attn(q[:, a:b], k, v, idx, None if g is None else g[:, a:b], q_pos0=a)
        assert torch.equal(o, o_w[:, a:b]), (a, b)
    assert sala.get_device_error() == 0


@pytest.mark.parametrize("T,Hq,Hkv,D,topk,score,cuts", [
    # fused tensor-core selection; windows not aligned to blocks or 128-row items
    (64 * 150 + 45, 32, 2, 128, 64, "group_sum", [0, 1000, 5003, 9000, None]),
    # topk > 64: the score-scratch selection
    (64 * 200 + 9, 16, 2, 128, 100, "group_sum", [0, 4321, 4322, None]),
    # per-head softmax selection, head_dim 64
    (64 * 90 + 31, 16, 1, 64, 32, "head_softmax", [0, 64 * 45 + 7, None]),
    # windows shorter than the dense threshold and a one-row window at the end
    (64 * 80, 8, 2, 128, 16, "group_sum", [0, 63, 64, 4000, 64 * 80 - 1, None]),
])
def test_row_windows_equal_whole_sequence(T, Hq, Hkv, D, topk, score, cuts):
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=900 + T, device=DEV, gate=True)
    _windows_match_whole(s, [T if c is None else c for c in cuts], topk=topk, score=score)


def test_row_windows_batched_strided():
    """Two sequences, q / k / v / g as strided views of wider tensors."""
    B, T, Hq, Hkv, D = 2, 64 * 70 + 13, 16, 2, 128
    s = inputs.sparse_inputs(B, T, Hq, Hkv, D, seed=941, device=DEV, gate=True)
    wide = lambda x: torch.cat([x, torch.zeros_like(x)], dim=2)[:, :, :x.shape[2]]
    s = inputs.SparseInputs(wide(s.q), wide(s.k), wide(s.v), wide(s.g))
    assert not s.q.is_contiguous()
    _windows_match_whole(s, [0, 2222, T], topk=32, n_local=3)


def test_row_window_against_oracle():
    T, Hq, Hkv, D, topk = 64 * 96 + 20, 16, 2, 128, 24
    a, b = 64 * 40 + 33, 64 * 70 + 2
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=955, gate=True)
    dq, dk, dv, dg = (x.cuda() for x in (s.q, s.k, s.v, s.g))
    idx = sala.sparse_select(dq[:, a:b], dk, topk=topk, q_pos0=a)
    rows = np.arange(a, b)
    ref, gap, sc = oracle.sparse_select(_np(s.q[:, a:b]), _np(s.k), topk=topk, rows=rows,
                                        want_scores=True)
    check_index_sets(idx.cpu().numpy(), ref, gap, sc, rows, topk=topk)
    o = sala.sparse_attn(dq[:, a:b], dk, dv, idx, dg[:, a:b], q_pos0=a)
    yref = oracle.attention(_np(s.q[:, a:b]), _np(s.k), _np(s.v), _np(s.g[:, a:b]),
                            idx=idx.cpu().numpy(), rows=rows)
    assert rel_err(_np(o), yref, True) <= TOL_BF16
    assert sala.get_device_error() == 0


def test_row_windows_full_size():
    """T = 131072, 32q/2kv D128, top-64: the four windows of a four-way query split equal
    the whole-sequence selection and attention bit for bit."""
    T, Hq, Hkv, D = 131072, 32, 2, 128
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=1004, device=DEV, gate=True)
    _windows_match_whole(s, [0, T // 4, T // 2, 3 * T // 4, T])


def test_query_parallel_layer_single_rank_group():
    """The host logic with three emulated ranks (the all-gather already done: every rank
    gets the whole k and v) and the public call on a one-rank NCCL group both equal the
    plain whole-sequence layer bit for bit."""
    import os
    import socket

    import torch.distributed as dist

    from sparse_attention_long_lightning_b200.seqpar import (segment_offsets,
                                                              sparse_layer_qrange,
                                                              sparse_layer_query_parallel)
    T, Hq, Hkv, D = 64 * 60 + 29, 32, 2, 128
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=977, device=DEV, gate=True)
    y_ref = sala.sparse_attn(s.q, s.k, s.v, sala.sparse_select(s.q, s.k, topk=16), s.g)
    lens = [1500, 1000, T - 2500]
    offs = segment_offsets(lens)
    parts = []
    for r in range(3):
        lo, hi = offs[r], offs[r] + lens[r]
        parts.append(sparse_layer_qrange(
            s.q[:, lo:hi], s.k[:, lo:hi], s.v[:, lo:hi], s.g[:, lo:hi], rank=r, offsets=offs,
            gather_kv=lambda kk, vv: (s.k, s.v),
            select_fn=lambda qq, K, p: sala.sparse_select(qq, K, topk=16, q_pos0=p),
            attn_fn=lambda qq, K, V, idx, gg, p: sala.sparse_attn(qq, K, V, idx, gg, q_pos0=p)))
    assert torch.equal(torch.cat(parts, dim=1), y_ref)
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    os.environ["MASTER_ADDR"], os.environ["MASTER_PORT"] = "127.0.0.1", str(port)
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        y = sparse_layer_query_parallel(s.q, s.k, s.v, s.g, topk=16)
        assert torch.equal(y, y_ref)
    finally:
        dist.destroy_process_group()
    assert sala.get_device_error() == 0


def test_row_window_rejects_bad_windows():
    s = inputs.sparse_inputs(1, 640, 16, 2, 128, seed=3, device=DEV)
    with pytest.raises(ValueError):
        sala.sparse_select(s.q[:, :100], s.k)              # lengths differ, no q_pos0
    with pytest.raises(ValueError):
        sala.sparse_select(s.q[:, :100], s.k, q_pos0=600)  # window past the keys
    idx = sala.sparse_select(s.q[:, :0], s.k, q_pos0=640)  # empty window at the end
    assert idx.shape == (1, 2, 0, 67)
