"""GPU parity: sparse-layer decode (libsala) vs the fp64 oracle.

The decode step at position p is row p of the prefill computation over cache rows
0..p.  The selection is compared with the oracle's (bit-exact except near-ties); the
output is compared with the oracle's attention over the GPU's own selection, so a
near-tie in the selection cannot move the output check.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_long_lightning_b200 import inputs
from tests._parity import TOL_BF16, check_index_sets, rel_err, rel_err_bf16_pair

pytestmark = pytest.mark.gpu

sala = pytest.importorskip("sparse_attention_long_lightning_b200")
DEV = "cuda"
SALA_ERR_RANGE = 6


def _np(t):
    return t.detach().double().cpu().numpy()


def _data(B, Tmax, Hq, Hkv, D, seed):
    gen = inputs.generator(seed)
    q = inputs.randn((B, Hq, D), gen)
    g = inputs.randn((B, Hq, D), gen)
    k = inputs.randn((B, Tmax, Hkv, D), gen)
    v = inputs.randn((B, Tmax, Hkv, D), gen)
    return q, g, k, v


def _check_step(q, g, k, v, pos, y, idx, topk=64, n_init=1, n_local=2):
    """Selection vs the oracle's, output vs the oracle's attention over the GPU selection."""
    qn, kn, vn = _np(q), _np(k), _np(v)
    gn = None if g is None else _np(g)
    _, ref_idx, gap, sc = oracle.sparse_decode(qn, kn, vn, pos, gn, topk=topk, n_init=n_init,
                                               n_local=n_local, want_scores=True)
    gi = idx.cpu().numpy()
    check_index_sets(gi[:, :, None, :], ref_idx[:, :, None, :], gap[:, :, None],
                     sc[:, :, None, :], np.asarray(pos)[:, None, None], topk=topk,
                     n_init=n_init, n_local=n_local)
    for b, p in enumerate(pos):
        want = oracle.attention(qn[b][None, None], kn[b:b + 1, :p + 1], vn[b:b + 1, :p + 1],
                                None if gn is None else gn[b][None, None],
                                idx=gi[b][:, None, :], rows=[p])[0, 0]
        err = rel_err(_np(y[b]), want, bf16_out=True)
        assert err <= TOL_BF16, (b, p, err)


@pytest.mark.parametrize("Hq,Hkv,D,gate", [(32, 2, 128, True), (8, 2, 64, False),
                                           (16, 1, 128, True)])
def test_decode_positions(Hq, Hkv, D, gate):
    """Positions before any candidate, at block ends (the step completes a block mean)
    and mid-block, in one batch."""
    Tmax = 64 * 48
    pos_l = [0, 63, 64 * 5 + 10, 64 * 20 + 63, 64 * 40 + 31, Tmax - 1]
    B = len(pos_l)
    q, g, k, v = _data(B, Tmax, Hq, Hkv, D, seed=Hq * 7 + D)
    q, g, k, v = q.to(DEV), (g.to(DEV) if gate else None), k.to(DEV), v.to(DEV)
    kbar = sala.sparse_block_means(k, kbar_blocks=Tmax // 64)
    # the means of the blocks that these steps complete must come from the step itself
    for b, p in enumerate(pos_l):
        if (p + 1) % 64 == 0:
            kbar[b, p // 64] = float("nan")
    pos = torch.tensor(pos_l, dtype=torch.int32, device=DEV)
    idx = torch.empty((B, Hkv, 67), dtype=torch.int32, device=DEV)
    y = sala.sparse_decode(q, k, v, kbar, pos, g, idx_out=idx)
    assert sala.get_device_error() == 0
    _check_step(q, g, k, v, pos_l, y, idx)
    full = sala.sparse_block_means(k, kbar_blocks=Tmax // 64)
    for b, p in enumerate(pos_l):
        if (p + 1) % 64 == 0:
            assert torch.equal(kbar[b, p // 64], full[b, p // 64])


def test_decode_wider_windows():
    """n_init = 2, n_local = 6, topk = 20: selection and output against the oracle."""
    Tmax, Hq, Hkv, D = 64 * 64, 32, 2, 128
    pos_l = [64 * 3, 64 * 9 + 63, 64 * 40 + 5, Tmax - 1]
    B = len(pos_l)
    q, g, k, v = _data(B, Tmax, Hq, Hkv, D, seed=409)
    q, g, k, v = q.to(DEV), g.to(DEV), k.to(DEV), v.to(DEV)
    kbar = sala.sparse_block_means(k)
    pos = torch.tensor(pos_l, dtype=torch.int32, device=DEV)
    idx = torch.empty((B, Hkv, 28), dtype=torch.int32, device=DEV)
    y = sala.sparse_decode(q, k, v, kbar, pos, g, topk=20, n_init=2, n_local=6, idx_out=idx)
    assert sala.get_device_error() == 0
    _check_step(q, g, k, v, pos_l, y, idx, topk=20, n_init=2, n_local=6)


def test_decode_steps_continue_a_prefilled_cache():
    """70 consecutive steps after a 1970-token prefill, crossing two block ends: every
    step against the oracle, then the block-mean cache against the oracle's means."""
    B, Hq, Hkv, D, Tmax, T0, steps = 2, 32, 2, 128, 64 * 34, 1970, 70
    q_all, g_all, k, v = _data(B, Tmax, Hq, Hkv, D, seed=404)
    gen = inputs.generator(405)
    qs = inputs.randn((steps, B, Hq, D), gen).to(DEV)
    gs = inputs.randn((steps, B, Hq, D), gen).to(DEV)
    k, v = k.to(DEV), v.to(DEV)
    kbar = torch.zeros((B, Tmax // 64, Hkv, D), dtype=torch.float32, device=DEV)
    sala.sparse_block_means(k[:, :T0], kbar)
    idx = torch.empty((B, Hkv, 67), dtype=torch.int32, device=DEV)
    ws = torch.empty(sala.sparse_decode_workspace(B, Tmax, Hq, Hkv, D, 67), dtype=torch.uint8,
                     device=DEV)
    for s in range(steps):
        p = T0 + s
        pos = torch.full((B,), p, dtype=torch.int32, device=DEV)
        y = sala.sparse_decode(qs[s], k, v, kbar, pos, gs[s], idx_out=idx, workspace=ws)
        if s % 7 == 0 or (p + 1) % 64 == 0 or s == steps - 1:
            _check_step(qs[s], gs[s], k, v, [p] * B, y, idx)
    assert sala.get_device_error() == 0
    T_end = T0 + steps
    nb = T_end // 64
    want = oracle.block_means(_np(k[:, :T_end]))
    got = kbar[:, :nb].double().cpu().numpy()
    assert np.abs(got - want).max() <= 1e-6 * np.abs(want).max()
    assert torch.equal(kbar[:, :nb], sala.sparse_block_means(k[:, :T_end])[:, :nb])


def test_decode_matches_prefill_rows():
    """Decode at p with the prefill's query row p reproduces the prefill output row p."""
    T, Hq, Hkv, D = 64 * 40 + 17, 32, 2, 128
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=406, device=DEV, gate=True)
    idx_pf = sala.sparse_select(s.q, s.k)
    y_pf = sala.sparse_attn(s.q, s.k, s.v, idx_pf, s.g)
    Tmax = (T + 63) // 64 * 64
    k = torch.zeros((1, Tmax, Hkv, D), dtype=torch.bfloat16, device=DEV)
    v = torch.zeros_like(k)
    k[:, :T], v[:, :T] = s.k, s.v
    kbar = sala.sparse_block_means(k[:, :T], kbar_blocks=Tmax // 64)
    rows = [5, 64 * 3 + 2, 64 * 17 + 63, 64 * 30 + 40, T - 1]
    _, gap, sc = oracle.sparse_select(_np(s.q[:, rows]), _np(s.k), rows=rows, want_scores=True)
    idx = torch.empty((1, Hkv, 67), dtype=torch.int32, device=DEV)
    for r, p in enumerate(rows):
        pos = torch.tensor([p], dtype=torch.int32, device=DEV)
        y = sala.sparse_decode(s.q[:, p], k, v, kbar.clone(), pos, s.g[:, p], idx_out=idx)
        # the prefill's selection stands in for the oracle's here: both sides are the GPU's,
        # so the oracle's gap and scores decide which rows may differ and how
        check_index_sets(idx.cpu().numpy()[:, :, None], idx_pf[:, :, p:p + 1].cpu().numpy(),
                         gap[:, :, r:r + 1], sc[:, :, r:r + 1], p, topk=64)
        if torch.equal(idx[0], idx_pf[0, :, p]):
            assert rel_err_bf16_pair(_np(y[0]), _np(y_pf[0, p])) <= TOL_BF16


def test_decode_full_context_sampled():
    """T = 131072 caches (the sparse layer's prefill size): the last position and one
    just past a block end, against the oracle."""
    B, Hq, Hkv, D, Tmax = 2, 32, 2, 128, 131072
    q, g, k, v = _data(B, Tmax, Hq, Hkv, D, seed=407)
    q, g, k, v = q.to(DEV), g.to(DEV), k.to(DEV), v.to(DEV)
    kbar = sala.sparse_block_means(k)
    pos_l = [Tmax - 1, Tmax - 64 * 7 + 3]
    pos = torch.tensor(pos_l, dtype=torch.int32, device=DEV)
    idx = torch.empty((B, Hkv, 67), dtype=torch.int32, device=DEV)
    y = sala.sparse_decode(q, k, v, kbar, pos, g, idx_out=idx)
    assert sala.get_device_error() == 0
    _check_step(q, g, k, v, pos_l, y, idx)


def test_decode_position_outside_cache_raises_range():
    """A position outside [0, Tmax) is caught by the kernels' own check: that sequence
    is skipped and the device error word reads RANGE; the others are still computed."""
    B, Hq, Hkv, D, Tmax = 3, 16, 2, 128, 64 * 8
    q, g, k, v = _data(B, Tmax, Hq, Hkv, D, seed=408)
    q, g, k, v = q.to(DEV), g.to(DEV), k.to(DEV), v.to(DEV)
    kbar = sala.sparse_block_means(k)
    pos_l = [100, Tmax, -1]
    pos = torch.tensor(pos_l, dtype=torch.int32, device=DEV)
    idx = torch.empty((B, Hkv, 67), dtype=torch.int32, device=DEV)
    y = sala.sparse_decode(q, k, v, kbar, pos, g, idx_out=idx)
    assert sala.get_device_error() == SALA_ERR_RANGE
    _check_step(q[:1], g[:1], k[:1], v[:1], pos_l[:1], y[:1], idx[:1])
    assert sala.get_device_error() == 0
