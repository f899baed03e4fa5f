"""GPU parity: block selection and block-sparse attention (libsala) vs the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_long_lightning_b200 import inputs
from tests._parity import TOL_BF16, check_index_sets, raw_rel_err, rel_err

pytestmark = pytest.mark.gpu

sala = pytest.importorskip("sparse_attention_long_lightning_b200")
DEV = "cuda"


def _np(t):
    return t.detach().double().cpu().numpy()


def _sampled_rows(T, n_mid=1024, seed=0):
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(256, T - 256), size=min(n_mid, T - 512), replace=False)
    return np.unique(np.concatenate([np.arange(256), mid, np.arange(T - 256, T)]))


@pytest.mark.parametrize("T,Hq,Hkv,D,topk", [
    (64 * 20 + 17, 16, 2, 128, 4), (64 * 40, 32, 2, 128, 8), (64 * 9 + 63, 8, 1, 64, 3),
    (50, 16, 1, 128, 64), (64 * 70 + 5, 16, 1, 128, 64), (4288, 16, 2, 64, 64)])
def test_select_small(T, Hq, Hkv, D, topk):
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=T + Hq)
    idx = sala.sparse_select(s.q.cuda(), s.k.cuda(), topk=topk)
    ref, gap, sc = oracle.sparse_select(_np(s.q), _np(s.k), topk=topk, want_scores=True)
    check_index_sets(idx.cpu().numpy(), ref, gap, sc, np.arange(T), topk=topk)


def test_select_topk_above_fused_limit():
    """topk > 64 takes the score-scratch path (scores in fp32, per-row radix select)."""
    T, Hq, Hkv, D, topk = 64 * 200 + 9, 16, 2, 128, 100
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=77)
    idx = sala.sparse_select(s.q.cuda(), s.k.cuda(), topk=topk)
    ref, gap, sc = oracle.sparse_select(_np(s.q), _np(s.k), topk=topk, want_scores=True)
    check_index_sets(idx.cpu().numpy(), ref, gap, sc, np.arange(T), topk=topk)


def test_select_exact_ties_take_smaller_blocks():
    """Every block holds the same keys, so all candidate scores of a row are equal:
    the selection must be the topk smallest candidate indices, exactly."""
    T, Hq, Hkv, D, topk = 64 * 300 + 10, 16, 2, 128, 64
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=78)
    k = s.k[:, :64].repeat(1, (T + 63) // 64, 1, 1)[:, :T].contiguous()
    idx = sala.sparse_select(s.q.cuda(), k.cuda(), topk=topk).cpu().numpy()
    ref, _ = oracle.sparse_select(_np(s.q), _np(k), topk=topk)
    assert np.array_equal(idx, ref)


@pytest.mark.parametrize("n_init,n_local", [(1, 8), (2, 5)])
def test_select_and_attn_wider_windows(n_init, n_local):
    """A larger local window and more init blocks (the selection rule's window sizes are
    parameters): selection and attention against the oracle."""
    T, Hq, Hkv, D, topk = 64 * 150 + 40, 16, 2, 128, 16
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=80 + n_local, gate=True)
    q, k, v, g = (t.cuda() for t in (s.q, s.k, s.v, s.g))
    idx = sala.sparse_select(q, k, topk=topk, n_init=n_init, n_local=n_local)
    rows = _sampled_rows(T, n_mid=600, seed=6)
    ref, gap, sc = oracle.sparse_select(_np(s.q[:, rows]), _np(s.k), topk=topk, n_init=n_init,
                                        n_local=n_local, rows=rows, want_scores=True)
    check_index_sets(idx.cpu().numpy()[:, :, rows], ref, gap, sc, rows, topk=topk,
                     n_init=n_init, n_local=n_local)
    y = sala.sparse_attn(q, k, v, idx, g)
    want = oracle.attention(_np(s.q[:, rows]), _np(s.k), _np(s.v), _np(s.g[:, rows]),
                            idx=idx.cpu().numpy()[:, :, rows], rows=rows)
    assert rel_err(_np(y[:, rows]), want, bf16_out=True) <= TOL_BF16


def test_select_heavy_tailed_scores():
    """Ten blocks whose keys are a large constant vector: every row's scores are far from
    normal (ten extreme values on one side), the case a distribution-based shortcut
    would get wrong; the selection must still match the oracle."""
    T, Hq, Hkv, D, topk = 64 * 600 + 21, 16, 2, 128, 64
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=79)
    k = s.k.clone()
    k[:, 64 * 5:64 * 15] = 30.0
    idx = sala.sparse_select(s.q.cuda(), k.cuda(), topk=topk)
    rows = _sampled_rows(T, n_mid=1500, seed=5)
    ref, gap, sc = oracle.sparse_select(_np(s.q[:, rows]), _np(k), topk=topk, rows=rows,
                                        want_scores=True)
    check_index_sets(idx.cpu().numpy()[:, :, rows], ref, gap, sc, rows, topk=topk)


def test_select_batched_strided():
    """B = 2 with q, k as views of a packed tensor (non-contiguous strides)."""
    B, T, Hq, Hkv, D = 2, 64 * 13 + 30, 16, 2, 128
    gen = inputs.generator(31)
    packed = inputs.randn((B, T, Hq + 2 * Hkv, D), gen)
    q, k = packed[:, :, :Hq], packed[:, :, Hq:Hq + Hkv]
    d = packed.cuda()
    idx = sala.sparse_select(d[:, :, :Hq], d[:, :, Hq:Hq + Hkv], topk=5)
    ref, gap, sc = oracle.sparse_select(_np(q), _np(k), topk=5, want_scores=True)
    check_index_sets(idx.cpu().numpy(), ref, gap, sc, np.arange(T), topk=5)


@pytest.mark.parametrize("T,Hq,Hkv,D,topk,gate", [
    (64 * 20 + 17, 16, 2, 128, 4, True), (64 * 9 + 63, 8, 1, 64, 3, False),
    (33, 16, 1, 128, 64, True), (64 * 12, 16, 1, 128, 64, False),
    (64 * 9 + 63, 8, 1, 128, 3, True), (64 * 30 + 1, 24, 2, 128, 5, True)])
def test_sparse_attn_small(T, Hq, Hkv, D, topk, gate):
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=3 * T + D, gate=gate)
    dq, dk, dv = s.q.cuda(), s.k.cuda(), s.v.cuda()
    dg = s.g.cuda() if gate else None
    idx = sala.sparse_select(dq, dk, topk=topk)
    o = sala.sparse_attn(dq, dk, dv, idx, dg)
    ref = oracle.attention(_np(s.q), _np(s.k), _np(s.v), _np(s.g) if gate else None,
                           idx=idx.cpu().numpy())
    assert rel_err(_np(o), ref, True) <= TOL_BF16
    assert sala.get_device_error() == 0


def test_sparse_attn_unordered_and_shared_selections():
    """The attention kernel merges the block lists of 8 consecutive query rows and reads a
    block they share once: rows whose lists are in arbitrary order (entries shuffled,
    -1 padding included), and rows of a query block that all pick the same blocks, both
    against the oracle (which does not depend on the order of a row's entries)."""
    T, Hq, Hkv, D = 64 * 50 + 13, 16, 2, 128
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=90, gate=True)
    q, k, v, g = (t.cuda() for t in (s.q, s.k, s.v, s.g))
    idx = sala.sparse_select(q, k, topk=16).cpu().numpy()
    rows = np.unique(np.concatenate([np.arange(0, T, 5), np.arange(T - 70, T)]))
    shuffled = np.random.default_rng(9).permuted(idx, axis=-1)
    same = idx.copy()
    for t in range(T):  # every row takes the list of the last row of its query block
        same[:, :, t] = idx[:, :, min(T - 1, t // 64 * 64 + 63)]
    for sel in (shuffled, same):
        o = sala.sparse_attn(q, k, v, torch.from_numpy(np.ascontiguousarray(sel)).cuda(), g)
        assert sala.get_device_error() == 0
        want = oracle.attention(_np(s.q[:, rows]), _np(s.k), _np(s.v), _np(s.g[:, rows]),
                                idx=sel[:, :, rows], rows=rows)
        assert rel_err(_np(o[:, rows]), want, True) <= TOL_BF16


def test_sparse_equals_dense_at_budget_length():
    """T = 67 * 64 = 4288: every causal block is selected, so the sparse path is
    dense causal attention (the dense fallback)."""
    T, Hq, Hkv, D = 4288, 16, 1, 128
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=4288)
    dq, dk, dv = s.q.cuda(), s.k.cuda(), s.v.cuda()
    o = sala.sparse_attn(dq, dk, dv, sala.sparse_select(dq, dk))
    rows = _sampled_rows(T, 512)
    ref = oracle.attention(_np(s.q[:, rows]), _np(s.k), _np(s.v), rows=rows)
    assert rel_err(_np(o[:, rows]), ref, True) <= TOL_BF16


def test_sparse_attn_empty_and_partial_rows():
    """Rows with no entries give zeros; entries beyond the row's position are skipped."""
    T, Hq, Hkv, D = 200, 16, 1, 128
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=5)
    idx = torch.full((1, Hkv, T, 3), -1, dtype=torch.int32)
    idx[0, 0, 100:, 0] = 1           # block 1 = keys 64..127
    idx[0, 0, 150:, 1] = 3           # block 3 (keys 192..199) only reachable from t >= 192
    o = sala.sparse_attn(s.q.cuda(), s.k.cuda(), s.v.cuda(), idx.cuda())
    ref = oracle.attention(_np(s.q), _np(s.k), _np(s.v), idx=idx.numpy())
    out = _np(o)
    assert np.all(out[:, :100] == 0.0)
    assert rel_err(out[:, 100:], ref[:, 100:], True) <= TOL_BF16


def test_sparse_128k_full_size_sampled_rows():
    """Sparse prefill B1 T131072 Hq32 Hkv2 D128 (seed 1004) in the benchmark's launch
    configuration: selection compared on sampled rows (first/last 256 and 1024
    spread rows, both KV heads), attention on the same rows with the GPU's
    selection fed to the oracle."""
    T, Hq, Hkv, D = 131072, 32, 2, 128
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=1004, device=DEV, gate=True)
    idx = sala.sparse_select(s.q, s.k)
    o = sala.sparse_attn(s.q, s.k, s.v, idx, s.g)
    rows = _sampled_rows(T, 1024, seed=1)
    q_rows = _np(s.q[:, rows])
    k_np, v_np = _np(s.k), _np(s.v)
    ref_idx, gap, sc = oracle.sparse_select(q_rows, k_np, rows=rows, T=T, want_scores=True)
    gi = idx[:, :, rows].cpu().numpy()
    ndiff, nrow = check_index_sets(gi, ref_idx, gap, sc, rows, topk=64)
    ref_o = oracle.attention(q_rows, k_np, v_np, _np(s.g[:, rows]), idx=gi, rows=rows)
    e = rel_err(_np(o[:, rows]), ref_o, True)
    print(f"128k sparse: index rows differing at near-ties {ndiff}/{nrow}; attn {e:.3e} "
          f"(raw {raw_rel_err(_np(o[:, rows]), ref_o):.3e})")
    assert e <= TOL_BF16
    assert sala.get_device_error() == 0


def test_sparse_1m_full_size_sampled_rows():
    """One sparse layer of the 1M-token hybrid stack: B1 T1048576 Hq32 Hkv2 D128 (seed
    1011), selection (16383 candidate blocks per late row) and attention compared on
    sampled rows of both KV heads (first/last 256 rows and 256 spread rows)."""
    T, Hq, Hkv, D = 1 << 20, 32, 2, 128
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=1011, device=DEV, gate=True)
    idx = sala.sparse_select(s.q, s.k)
    o = sala.sparse_attn(s.q, s.k, s.v, idx, s.g)
    rows = _sampled_rows(T, 256, seed=5)
    q_rows = _np(s.q[:, rows])
    k_np, v_np = _np(s.k), _np(s.v)
    ref_idx, gap, sc = oracle.sparse_select(q_rows, k_np, rows=rows, T=T, want_scores=True)
    gi = idx[:, :, rows].cpu().numpy()
    ndiff, nrow = check_index_sets(gi, ref_idx, gap, sc, rows, topk=64)
    ref_o = oracle.attention(q_rows, k_np, v_np, _np(s.g[:, rows]), idx=gi, rows=rows)
    e = rel_err(_np(o[:, rows]), ref_o, True)
    print(f"1m sparse: index rows differing at near-ties {ndiff}/{nrow}; attn {e:.3e}")
    assert e <= TOL_BF16
    assert sala.get_device_error() == 0


def test_bounded_wait_reports_timeout():
    """A device wait that can never complete gives up after its cycle budget and
    reports SALA_ERR_TIMEOUT through the device error word; the context stays usable."""
    sala.get_device_error()
    sala.selftest_wait_timeout(20_000_000)
    assert sala.get_device_error() == 4
    assert sala.get_device_error() == 0
    # the GPU still computes correctly afterwards
    T, Hq, Hkv, D = 200, 16, 1, 128
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=8)
    idx = sala.sparse_select(s.q.cuda(), s.k.cuda(), topk=2)
    o = sala.sparse_attn(s.q.cuda(), s.k.cuda(), s.v.cuda(), idx)
    ref = oracle.attention(_np(s.q), _np(s.k), _np(s.v), idx=idx.cpu().numpy())
    assert rel_err(_np(o), ref, True) <= TOL_BF16


def test_sparse_kvhead_parallel_single_rank_group():
    """The public KV-head-parallel call on a one-rank NCCL group (all heads on this rank,
    outputs all-gathered) is the plain selection + attention, bit for bit; and a rank's
    share computed on head views equals the same heads of the full layer."""
    import os
    import socket

    import torch.distributed as dist

    from sparse_attention_long_lightning_b200.seqpar import (sparse_layer_headpar,
                                                              sparse_layer_kvhead_parallel)
    T, Hq, Hkv, D = 64 * 30 + 11, 32, 2, 128
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=818, device=DEV, gate=True)
    y_ref = sala.sparse_attn(s.q, s.k, s.v, sala.sparse_select(s.q, s.k, topk=16), s.g)
    # rank 1 of 2 computed locally: KV head 1 and query heads 16..31, from views
    y1 = sparse_layer_headpar(s.q, s.k, s.v, s.g, rank=1, world=2,
                              select_fn=lambda qq, kk: sala.sparse_select(qq, kk, topk=16),
                              attn_fn=lambda qq, kk, vv, idx, gg: sala.sparse_attn(qq, kk, vv,
                                                                                   idx, gg))
    assert torch.equal(y1, y_ref[:, :, 16:])
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    os.environ["MASTER_ADDR"], os.environ["MASTER_PORT"] = "127.0.0.1", str(port)
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        y = sparse_layer_kvhead_parallel(s.q, s.k, s.v, s.g, topk=16)
        assert torch.equal(y, y_ref)
    finally:
        dist.destroy_process_group()
    assert sala.get_device_error() == 0


@pytest.mark.parametrize("T", [1, 63, 64, 65, 127, 4288, 4289])
def test_select_and_attn_edge_lengths(T):
    """Sequence lengths at block and budget edges (one token; one block -1, 0, +1; the
    dense-fallback limit 67 x 64 and one past it), two sequences, gated, selection and
    attention against the oracle."""
    B, Hq, Hkv, D, topk = 2, 16, 2, 128, 64
    s = inputs.sparse_inputs(B, T, Hq, Hkv, D, seed=700 + T, gate=True)
    dq, dk, dv, dg = (x.cuda() for x in (s.q, s.k, s.v, s.g))
    idx = sala.sparse_select(dq, dk, topk=topk)
    rows = np.arange(T) if T <= 512 else _sampled_rows(T, n_mid=256, seed=T)
    ref, gap, sc = oracle.sparse_select(_np(s.q[:, rows]), _np(s.k), topk=topk, rows=rows,
                                        want_scores=True)
    check_index_sets(idx.cpu().numpy()[:, :, rows], ref, gap, sc, rows, topk=topk)
    o = sala.sparse_attn(dq, dk, dv, idx, dg)
    want = oracle.attention(_np(s.q[:, rows]), _np(s.k), _np(s.v), _np(s.g[:, rows]),
                            idx=idx.cpu().numpy()[:, :, rows], rows=rows)
    assert rel_err(_np(o[:, rows]), want, True) <= TOL_BF16
    assert sala.get_device_error() == 0
