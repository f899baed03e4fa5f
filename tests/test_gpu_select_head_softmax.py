"""GPU parity: per-head softmax-normalised block selection (libsala) vs the fp64 oracle.

The GPU computes the scores in fp32 (exact products, expf, IEEE division, fp32 sums over
up to a few thousand candidates: relative error ~1e-6), so index sets must be
bit-exact except in rows whose oracle topk-th and (topk+1)-th scores differ by less
than 1e-5 of the topk-th score; there the sets may differ only by near-tied members.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_long_lightning_b200 import inputs
from tests._parity import check_index_sets

pytestmark = pytest.mark.gpu

sala = pytest.importorskip("sparse_attention_long_lightning_b200")
DEV = "cuda"
REL_BAND = 1e-5


def _np(t):
    return t.detach().double().cpu().numpy()


def _band(sc, topk):
    """Per-row tie band: REL_BAND times the oracle's topk-th score (0 when a row has
    no more than topk candidates; those rows have an infinite gap and must match)."""
    s = np.where(np.isnan(sc), -np.inf, sc)
    s = -np.sort(-s, axis=-1)
    kth = s[..., topk - 1] if s.shape[-1] >= topk else np.full(s.shape[:-1], -np.inf)
    return REL_BAND * np.where(np.isfinite(kth), np.abs(kth), 0.0)


def _check(idx_gpu, q, k, topk, rows=None, **kw):
    qn = _np(q) if rows is None else _np(q[:, rows])
    ref, gap, sc = oracle.sparse_select(qn, _np(k), topk=topk, rows=rows, want_scores=True,
                                        score="head_softmax", **kw)
    got = idx_gpu if rows is None else idx_gpu[:, :, rows]
    t = np.arange(q.shape[1]) if rows is None else np.asarray(rows)
    win = {key: kw[key] for key in ("n_init", "n_local") if key in kw}
    return check_index_sets(got, ref, gap, sc, t, topk=topk, tie_band=_band(sc, topk), **win)


@pytest.mark.parametrize("T,Hq,Hkv,D,topk", [
    (64 * 40 + 17, 32, 2, 128, 16),   # G = 16, ragged tail
    (64 * 33 + 5, 8, 2, 64, 8),       # G = 4, D = 64
    (64 * 25 + 40, 4, 4, 128, 6),     # G = 1
    (64 * 20 + 3, 64, 2, 128, 8),     # G = 32
    (64 * 90, 16, 8, 128, 64),        # G = 2, topk 64
    (64 * 12 + 9, 16, 2, 128, 64),    # every row within budget: all causal blocks
])
def test_head_softmax_select_small(T, Hq, Hkv, D, topk):
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=T + 3 * Hq)
    idx = sala.sparse_select(s.q.to(DEV), s.k.to(DEV), topk=topk, score="head_softmax")
    assert sala.get_device_error() == 0
    _check(idx.cpu().numpy(), s.q, s.k, topk)


def test_head_softmax_select_wider_windows_batched():
    """n_init = 2, n_local = 5, batch 2 with strided (non-contiguous) q and k."""
    B, T, Hq, Hkv, D, topk = 2, 64 * 50 + 21, 16, 2, 128, 12
    s = inputs.sparse_inputs(B, T, Hq, Hkv, D, seed=515)
    qb = torch.empty((B, T, Hq + 4, D), dtype=torch.bfloat16)
    kb = torch.empty((B, T, Hkv + 1, D), dtype=torch.bfloat16)
    qb[:, :, :Hq], kb[:, :, :Hkv] = s.q, s.k
    q, k = qb.to(DEV)[:, :, :Hq], kb.to(DEV)[:, :, :Hkv]
    idx = sala.sparse_select(q, k, topk=topk, n_init=2, n_local=5, score="head_softmax")
    assert sala.get_device_error() == 0
    _check(idx.cpu().numpy(), s.q, s.k, topk, n_init=2, n_local=5)


def test_head_softmax_select_128k_sampled_rows():
    """T = 131072, 32 query / 2 KV heads, topk 64 (the sparse layer's size): the full
    selection on the GPU, sampled rows (first, last, evenly spread) against the oracle."""
    T, Hq, Hkv, D, topk = 131072, 32, 2, 128, 64
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=1004, device=DEV)
    idx = sala.sparse_select(s.q, s.k, topk=topk, score="head_softmax").cpu().numpy()
    assert sala.get_device_error() == 0
    rows = np.unique(np.concatenate([np.arange(0, 4500, 499), np.linspace(4500, T - 1, 40)
                                     .astype(np.int64), [T - 1]]))
    _check(idx, s.q.cpu(), s.k.cpu(), topk, rows=rows.tolist(), T=T)
