"""Pins for the fp64 oracle (CPU only).

Each test ties an oracle routine to something other than itself: an algebraic
identity between independently written formulations, a closed form, an
invariant, brute-force enumeration, or a library routine (numpy / torch SDPA in
float64).  The mistakes these are meant to catch: a dropped term (initial
state, diagonal of the causal mask, a GQA head), a wrong sign or pairing in the
rotary embedding, a wrong frequency exponent, an off-by-one in block ranges,
a transposed operand in the state update, a reversed tie-break.
"""
import math

import numpy as np
import pytest
import torch

import oracle

RNG = np.random.default_rng(12345)


def _rand(*shape, rng=None):
    return (rng or RNG).standard_normal(shape)


# ----------------------------------------------------------------------------
# QK-normalisation and RoPE
# ----------------------------------------------------------------------------

def test_rmsnorm_closed_form():
    """At pos 0 the rotation is the identity, so qk_prep is RMSNorm alone:
    mean(y^2) = m / (m + eps) with m = mean(x^2), and y is parallel to x * w."""
    for D in (4, 64, 128):
        x = _rand(D)
        for eps in (0.0, 1e-6, 0.5):
            y = oracle.qk_prep(x, eps=eps, pos=0)
            m = np.mean(x * x)
            assert np.isclose(np.mean(y * y), m / (m + eps), rtol=1e-13)
            np.testing.assert_allclose(y, x / math.sqrt(m + eps), rtol=1e-13)
        w = _rand(D)
        y = oracle.qk_prep(x, w, eps=1e-6, pos=0)
        np.testing.assert_allclose(y, x * w / math.sqrt(np.mean(x * x) + 1e-6), rtol=1e-13)


def test_rope_basis_vectors_golden():
    """Rotate-half pairing on D=4, base 10000: pairs (0,2) and (1,3) with angular
    frequencies 1 and 10000^(-1/2) = 0.01.  Values derived by hand from the
    convention (tests/golden/rope_d4.txt records them)."""
    rows = []
    with open(__file__.replace("test_oracle_pins.py", "golden/rope_d4.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append([float(t) for t in line.split()])
    assert len(rows) == 4
    for basis, row in enumerate(rows):
        pos, expect = row[0], np.array(row[1:])
        x = np.zeros(4)
        x[basis] = 1.0
        # RMSNorm of a unit basis vector in D=4 scales it by 1/sqrt(1/4 + eps)
        y = oracle.qk_prep(x, eps=0.0, pos=pos) / 2.0
        np.testing.assert_allclose(y, expect, atol=1e-12)


def test_rope_relative_position_and_norm():
    """<R_m x, R_n y> depends only on m - n, and |R_m x| = |x| (after norm)."""
    D = 64
    x, y = _rand(D), _rand(D)
    for m, n, r in ((5, 2, 7), (0, 100, 3), (1000, 999, 123456)):
        a = oracle.qk_prep(x, pos=m) @ oracle.qk_prep(y, pos=n)
        b = oracle.qk_prep(x, pos=m + r) @ oracle.qk_prep(y, pos=n + r)
        assert abs(a - b) < 1e-9 * max(1.0, abs(a))
        z0 = oracle.qk_prep(x, pos=0)
        assert np.isclose(np.linalg.norm(oracle.qk_prep(x, pos=m)), np.linalg.norm(z0), rtol=1e-13)


def test_rope_frequency_exponent():
    """Pair i turns by pos * base^(-2i/D): the angle of (y_i, y_{i+D/2}) for the
    basis vector e_i pins the exponent (a -i/D or -2i/(D-2) variant fails)."""
    D, base, pos = 16, 10000.0, 3.0
    for i in range(D // 2):
        x = np.zeros(D)
        x[i] = 1.0
        y = oracle.qk_prep(x, eps=0.0, pos=pos, base=base)
        ang = math.atan2(y[i + D // 2], y[i])
        want = math.remainder(pos * base ** (-2.0 * i / D), 2 * math.pi)
        assert abs(ang - want) < 1e-12


# ----------------------------------------------------------------------------
# Lightning attention
# ----------------------------------------------------------------------------

def _lightning_case(B=2, T=37, H=3, D=8, seed=0, gate=True, s0=True, weights=True):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((B, T, H, D)) for _ in range(3))
    g = rng.standard_normal((B, T, H, D)) if gate else None
    S0 = rng.standard_normal((B, H, D, D)) * 0.3 if s0 else None
    qw = 1.0 + 0.1 * rng.standard_normal(D) if weights else None
    kw = 1.0 + 0.1 * rng.standard_normal(D) if weights else None
    return q, k, v, g, S0, qw, kw


@pytest.mark.parametrize("gate,s0,weights", [(True, True, True), (False, False, False),
                                             (True, False, False)])
def test_recurrent_equals_quadratic(gate, s0, weights):
    """Unrolling S_t = S_{t-1} + k_t v_t^T gives o_t = q_t^T S0 + sum_{s<=t}(q_t.k_s) v_s;
    the two routines share no accumulation code."""
    q, k, v, g, S0, qw, kw = _lightning_case(gate=gate, s0=s0, weights=weights)
    y1, _ = oracle.lightning_recurrent(q, k, v, g, S0, qw, kw, pos0=11)
    y2 = oracle.lightning_quadratic(q, k, v, g, S0, qw, kw, pos0=11)
    assert np.max(np.abs(y1 - y2)) <= 1e-12 * np.max(np.abs(y2))


@pytest.mark.parametrize("C", [1, 2, 3, 8, 16, 64, 37])
def test_chunked_equals_recurrent(C):
    """Chunked = recurrent for every chunk size, including ragged last chunks."""
    q, k, v, g, S0, qw, kw = _lightning_case(T=37)
    y1, S1 = oracle.lightning_recurrent(q, k, v, g, S0, qw, kw, pos0=3)
    y2, S2 = oracle.lightning_chunked(q, k, v, g, S0, qw, kw, chunk=C, pos0=3)
    assert np.max(np.abs(y1 - y2)) <= 1e-12 * np.max(np.abs(y1))
    assert np.max(np.abs(S1 - S2)) <= 1e-12 * np.max(np.abs(S1))


def test_final_state_closed_form():
    """S_T = S0 + sum_t khat_t v_t^T, checked with a numpy einsum over the
    normalised/rotated keys (a transposed update k^T v vs v^T k fails)."""
    q, k, v, g, S0, qw, kw = _lightning_case(T=20, D=8)
    _, S = oracle.lightning_recurrent(q, k, v, g, S0, qw, kw, pos0=2)
    B, T, H, D = q.shape
    kh = np.zeros_like(k)
    for b in range(B):
        for t in range(T):
            for h in range(H):
                kh[b, t, h] = oracle.qk_prep(k[b, t, h], kw, pos=2 + t)
    want = S0 + np.einsum("bthi,bthj->bhij", kh, v)
    np.testing.assert_allclose(S, want, rtol=1e-12, atol=1e-12)


def test_single_token_closed_form():
    """T=1, no initial state, q = k: o = |khat|^2 v = D*m/(m+eps) v (rotation keeps the
    norm), and the gate halves it at g = 0."""
    D = 16
    x = _rand(1, 1, 1, D)
    v = _rand(1, 1, 1, D)
    m = np.mean(x * x)
    y, _ = oracle.lightning_recurrent(x, x, v, pos0=77)
    np.testing.assert_allclose(y, D * m / (m + 1e-6) * v, rtol=1e-12)
    y, _ = oracle.lightning_recurrent(x, x, v, np.zeros_like(v), pos0=77)
    np.testing.assert_allclose(y, 0.5 * D * m / (m + 1e-6) * v, rtol=1e-12)


def test_zero_keys_read_initial_state():
    """k = 0 normalises to 0, so the state never changes and o_t = qhat_t^T S0."""
    q, k, v, g, S0, qw, kw = _lightning_case(T=9, gate=False)
    k[:] = 0.0
    y, S = oracle.lightning_recurrent(q, k, v, None, S0, None, None, pos0=0)
    np.testing.assert_allclose(S, S0, rtol=0, atol=0)
    B, T, H, D = q.shape
    for b in range(B):
        for t in range(T):
            for h in range(H):
                qh = oracle.qk_prep(q[b, t, h], pos=t)
                np.testing.assert_allclose(y[b, t, h], qh @ S0[b, h], rtol=1e-12, atol=1e-12)


def test_linear_in_values():
    """Without a gate the output is linear in v (and S0 = 0)."""
    q, k, v, _, _, qw, kw = _lightning_case(gate=False, s0=False)
    v2 = _rand(*v.shape)
    y1, _ = oracle.lightning_recurrent(q, k, v, qw=qw, kw=kw)
    y2, _ = oracle.lightning_recurrent(q, k, v2, qw=qw, kw=kw)
    y3, _ = oracle.lightning_recurrent(q, k, 2.0 * v - v2, qw=qw, kw=kw)
    np.testing.assert_allclose(y3, 2.0 * y1 - y2, rtol=1e-11, atol=1e-11)


def test_rows_subset_matches_full():
    q, k, v, g, S0, qw, kw = _lightning_case(T=30)
    yf, Sf = oracle.lightning_recurrent(q, k, v, g, S0, qw, kw, pos0=4)
    rows = [0, 5, 17, 29]
    yr, Sr = oracle.lightning_recurrent(q, k, v, g, S0, qw, kw, pos0=4, rows=rows)
    np.testing.assert_array_equal(yr, yf[:, rows])
    np.testing.assert_array_equal(Sr, Sf)


def test_segment_continuity():
    """prefill(T1) then prefill(T2) from its state at pos0 = T1 equals prefill(T1+T2)."""
    q, k, v, g, S0, qw, kw = _lightning_case(T=40)
    yf, Sf = oracle.lightning_recurrent(q, k, v, g, S0, qw, kw)
    ya, Sa = oracle.lightning_recurrent(q[:, :25], k[:, :25], v[:, :25], g[:, :25], S0, qw, kw)
    yb, Sb = oracle.lightning_recurrent(q[:, 25:], k[:, 25:], v[:, 25:], g[:, 25:], Sa, qw, kw,
                                        pos0=25)
    np.testing.assert_allclose(np.concatenate([ya, yb], axis=1), yf, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Sb, Sf, rtol=1e-12, atol=1e-12)


def test_decode_continues_prefill():
    """prefill(T) followed by a decode step at pos T equals row T of prefill(T+1)."""
    q, k, v, g, S0, qw, kw = _lightning_case(T=21)
    yf, Sf = oracle.lightning_recurrent(q, k, v, g, S0, qw, kw)
    _, S20 = oracle.lightning_recurrent(q[:, :20], k[:, :20], v[:, :20], g[:, :20], S0, qw, kw)
    B = q.shape[0]
    yd, Sd = oracle.lightning_decode(q[:, 20], k[:, 20], v[:, 20], g[:, 20], S20,
                                     np.full(B, 20), qw, kw)
    np.testing.assert_allclose(yd, yf[:, 20], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Sd, Sf, rtol=1e-12, atol=1e-12)


def test_decode_positions_per_batch():
    """Each batch entry uses its own position."""
    q, k, v, g, S0, qw, kw = _lightning_case(B=3, T=1)
    pos = np.array([0, 7, 1000])
    yd, _ = oracle.lightning_decode(q[:, 0], k[:, 0], v[:, 0], g[:, 0], S0, pos, qw, kw)
    for b in range(3):
        yr, _ = oracle.lightning_recurrent(q[b:b + 1], k[b:b + 1], v[b:b + 1], g[b:b + 1],
                                           S0[b:b + 1], qw, kw, pos0=int(pos[b]))
        np.testing.assert_allclose(yd[b], yr[0, 0], rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------
# Block selection
# ----------------------------------------------------------------------------

def test_block_means_closed_form():
    """k[t] = t: the mean of block j is 64 j + 31.5; a ragged tail block is dropped."""
    T = 64 * 5 + 17
    k = np.broadcast_to(np.arange(T, dtype=np.float64)[None, :, None, None], (1, T, 2, 3))
    km = oracle.block_means(k, 64)
    assert km.shape == (1, 5, 2, 3)
    np.testing.assert_array_equal(km[0, :, 0, 0], 64 * np.arange(5) + 31.5)


def test_block_means_match_numpy():
    k = _rand(2, 64 * 7 + 3, 2, 8)
    km = oracle.block_means(k, 64)
    want = k[:, : 64 * 7].reshape(2, 7, 64, 2, 8).mean(axis=2)
    np.testing.assert_allclose(km, want, rtol=1e-13, atol=1e-15)


def _check_structure(idx, T, blk, topk, n_init, n_local):
    B, Hkv, nrows, n_sel = idx.shape
    assert n_sel == n_init + topk + n_local
    for t in range(nrows):
        c = t // blk
        row = idx[0, 0, t]
        valid = row[row >= 0]
        assert np.all(row[len(valid):] == -1), "padding must be trailing -1"
        assert np.all(np.diff(valid) > 0), "sorted ascending, distinct"
        assert valid.max() <= c
        for j in range(min(n_init, c + 1)):
            assert j in valid
        for j in range(max(0, c - n_local + 1), c + 1):
            assert j in valid
        assert len(valid) == min(c + 1, n_sel)


def test_select_structure():
    T, blk = 64 * 9 + 5, 64
    q, k = _rand(1, T, 4, 8), _rand(1, T, 2, 8)
    idx, gap = oracle.sparse_select(q, k, blk=blk, topk=3, n_init=1, n_local=2)
    _check_structure(idx, T, blk, 3, 1, 2)


def test_select_planted_ranking():
    """Block j's keys all equal a_j * u and every query head is u: the score of j is
    a_j * Hgrp * |u|^2 / sqrt(D), so the top-k are the k largest a_j (closed form)."""
    blk, D, nb = 16, 8, 12
    T = blk * nb
    u = _rand(D)
    a = RNG.permutation(nb).astype(np.float64) + 1.0
    k = np.zeros((1, T, 1, D))
    for j in range(nb):
        k[0, j * blk:(j + 1) * blk, 0] = a[j] * u
    q = np.broadcast_to(u, (1, T, 4, D)).copy()
    idx, gap = oracle.sparse_select(q, k, blk=blk, topk=3, n_init=1, n_local=2)
    t = T - 1
    c = t // blk
    cands = list(range(1, c - 1))
    top = sorted(cands, key=lambda j: -a[j])[:3]
    want = sorted(set([0] + top + [c - 1, c]))
    got = [j for j in idx[0, 0, t] if j >= 0]
    assert got == want
    _, _, sc = oracle.sparse_select(q, k, blk=blk, topk=3, n_init=1, n_local=2, want_scores=True)
    for j in cands:
        assert np.isclose(sc[0, 0, t, j - 1], a[j] * 4 * (u @ u) / math.sqrt(D), rtol=1e-12)


def test_select_ties_prefer_smaller_block():
    """All candidate blocks identical: the top-k are the k smallest candidate indices."""
    blk, D, nb = 8, 4, 10
    T = blk * nb
    k = np.ones((1, T, 1, D))
    q = np.ones((1, T, 2, D))
    idx, gap = oracle.sparse_select(q, k, blk=blk, topk=2, n_init=1, n_local=2)
    got = [j for j in idx[0, 0, T - 1] if j >= 0]
    c = (T - 1) // blk
    assert got == [0, 1, 2, c - 1, c]
    assert gap[0, 0, T - 1] == 0.0


def test_select_bruteforce_subsets():
    """For small problems, enumerate every candidate subset of size topk; the chosen
    one must have the maximum total score (scores from a numpy sum-of-heads
    identity, (sum_h q_h) . kbar_j / sqrt(D), and numpy block means)."""
    import itertools

    rng = np.random.default_rng(7)
    blk, D, Hq, Hkv, topk = 8, 6, 4, 2, 3
    T = blk * 11 + 3
    q, k = rng.standard_normal((1, T, Hq, D)), rng.standard_normal((1, T, Hkv, D))
    idx, gap, sc = oracle.sparse_select(q, k, blk=blk, topk=topk, n_init=1, n_local=2,
                                        want_scores=True)
    nb = T // blk
    kbar = k[:, : nb * blk].reshape(1, nb, blk, Hkv, D).mean(axis=2)
    grp = Hq // Hkv
    for hk in range(Hkv):
        qs = q[0, :, hk * grp:(hk + 1) * grp].sum(axis=1)  # [T, D]
        for t in range(T):
            c = t // blk
            cands = list(range(1, c - 1))
            s = {j: qs[t] @ kbar[0, j, hk] / math.sqrt(D) for j in cands}
            for j in cands:
                assert np.isclose(sc[0, hk, t, j - 1], s[j], rtol=1e-12, atol=1e-12)
            if len(cands) <= topk:
                best = set(cands)
            else:
                best = max(itertools.combinations(cands, topk), key=lambda c_: sum(s[j] for j in c_))
                best = set(best)
            got = set(j for j in idx[0, hk, t] if j >= 0) - {0, c - 1, c}
            assert got == best, (hk, t)


# ----------------------------------------------------------------------------
# Attention (dense causal and block-sparse)
# ----------------------------------------------------------------------------

def _sdpa(q, k, v, mask):
    """torch scaled_dot_product_attention in float64 with an explicit boolean mask."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    grp = Hq // Hkv
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(np.repeat(k, grp, axis=2)).permute(0, 2, 1, 3)
    vt = torch.from_numpy(np.repeat(v, grp, axis=2)).permute(0, 2, 1, 3)
    m = torch.from_numpy(np.ascontiguousarray(mask))  # [B, Hq, T, T] bool
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m)
    return o.permute(0, 2, 1, 3).numpy()


def test_dense_attention_matches_sdpa():
    rng = np.random.default_rng(3)
    B, T, Hq, Hkv, D = 2, 29, 4, 2, 8
    q, k, v = (rng.standard_normal((B, T, h, D)) for h in (Hq, Hkv, Hkv))
    y = oracle.attention(q, k, v)
    mask = np.broadcast_to(np.tril(np.ones((T, T), dtype=bool)), (B, Hq, T, T))
    np.testing.assert_allclose(y, _sdpa(q, k, v, mask), rtol=1e-12, atol=1e-12)


def test_dense_attention_closed_forms():
    """Equal keys -> causal running mean of v; gate halves it at g = 0."""
    rng = np.random.default_rng(4)
    B, T, Hq, Hkv, D = 1, 13, 2, 1, 4
    q = rng.standard_normal((B, T, Hq, D))
    k = np.broadcast_to(rng.standard_normal(D), (B, T, Hkv, D)).copy()
    v = rng.standard_normal((B, T, Hkv, D))
    y = oracle.attention(q, k, v)
    cm = np.cumsum(v[0, :, 0], axis=0) / np.arange(1, T + 1)[:, None]
    for h in range(Hq):
        np.testing.assert_allclose(y[0, :, h], cm, rtol=1e-12)
    y = oracle.attention(q, k, v, np.zeros_like(q))
    np.testing.assert_allclose(y[0, :, 0], 0.5 * cm, rtol=1e-12)


def test_sparse_attention_matches_masked_sdpa():
    """Attention over selected blocks = SDPA with the block mask built from idx."""
    rng = np.random.default_rng(5)
    blk, B, Hq, Hkv, D = 8, 1, 4, 2, 8
    T = blk * 9 + 5
    q, k, v = (rng.standard_normal((B, T, h, D)) for h in (Hq, Hkv, Hkv))
    idx, _ = oracle.sparse_select(q, k, blk=blk, topk=2, n_init=1, n_local=2)
    y = oracle.attention(q, k, v, idx=idx, blk=blk)
    mask = np.zeros((B, Hq, T, T), dtype=bool)
    grp = Hq // Hkv
    for h in range(Hq):
        for t in range(T):
            for j in idx[0, h // grp, t]:
                if j >= 0:
                    mask[0, h, t, j * blk:min((j + 1) * blk, t + 1)] = True
    np.testing.assert_allclose(y, _sdpa(q, k, v, mask), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("T", [64 * 67, 300, 64])
def test_sparse_equals_dense_within_budget(T):
    """With T <= (n_init + topk + n_local) * blk every causal block is selected,
    so sparse attention is dense causal attention (the dense fallback)."""
    rng = np.random.default_rng(T)
    Hq, Hkv, D = 4, 2, 8
    q, k, v = (rng.standard_normal((1, T, h, D)) for h in (Hq, Hkv, Hkv))
    rows = np.unique(np.concatenate([np.arange(0, T, max(1, T // 40)), [T - 1]]))
    idx, _ = oracle.sparse_select(q[:, rows], k, rows=rows, T=T)
    ys = oracle.attention(q[:, rows], k, v, idx=idx, rows=rows)
    yd = oracle.attention(q[:, rows], k, v, rows=rows)
    np.testing.assert_allclose(ys, yd, rtol=1e-12, atol=1e-13)


def test_sparse_topk_covering_all_candidates_is_dense():
    rng = np.random.default_rng(9)
    blk, Hq, Hkv, D = 16, 2, 1, 4
    T = blk * 20
    q, k, v = (rng.standard_normal((1, T, h, D)) for h in (Hq, Hkv, Hkv))
    idx, gap = oracle.sparse_select(q, k, blk=blk, topk=18)
    assert np.all(np.isinf(gap))
    np.testing.assert_allclose(oracle.attention(q, k, v, idx=idx, blk=blk),
                               oracle.attention(q, k, v), rtol=1e-12, atol=1e-13)


def test_attention_rows_subset_and_empty_set():
    rng = np.random.default_rng(11)
    blk, Hq, Hkv, D = 8, 2, 1, 4
    T = 40
    q, k, v = (rng.standard_normal((1, T, h, D)) for h in (Hq, Hkv, Hkv))
    yf = oracle.attention(q, k, v)
    rows = [3, 17, 39]
    np.testing.assert_array_equal(oracle.attention(q[:, rows], k, v, rows=rows), yf[:, rows])
    empty = -np.ones((1, Hkv, T, 3), dtype=np.int32)
    assert np.all(oracle.attention(q, k, v, idx=empty, blk=blk) == 0.0)


# ----------------------------------------------------------------------------
# Sparse-layer decode (one query at position p over cache rows 0..p)
# ----------------------------------------------------------------------------

def _dense_row(q, k, v, p, g=None):
    """Plain numpy softmax attention of one query row over keys 0..p (GQA by repeat)."""
    Hq, D = q.shape
    Hkv = k.shape[1]
    grp = Hq // Hkv
    y = np.zeros((Hq, D))
    for h in range(Hq):
        s = k[:p + 1, h // grp] @ q[h] / math.sqrt(D)
        w = np.exp(s - s.max())
        y[h] = (w / w.sum()) @ v[:p + 1, h // grp]
        if g is not None:
            y[h] *= 1.0 / (1.0 + np.exp(-g[h]))
    return y


def test_decode_within_budget_is_dense_row():
    """While p + 1 <= (n_init + topk + n_local) * blk every causal block is chosen, so
    the decode output is the dense causal softmax row (numpy closed form)."""
    rng = np.random.default_rng(21)
    blk, Hq, Hkv, D, Tmax = 8, 4, 2, 8, 96
    q, g = rng.standard_normal((3, Hq, D)), rng.standard_normal((3, Hq, D))
    k, v = rng.standard_normal((3, Tmax, Hkv, D)), rng.standard_normal((3, Tmax, Hkv, D))
    pos = [0, 37, 8 * 5 - 1]  # topk 2 + init 1 + local 2 = 5 blocks of 8
    y, idx, _ = oracle.sparse_decode(q, k, v, pos, g, blk=blk, topk=2)
    for b, p in enumerate(pos):
        np.testing.assert_allclose(y[b], _dense_row(q[b], k[b], v[b], p, g[b]), rtol=1e-12,
                                   atol=1e-13)
        c = p // blk
        live = idx[b, 0][idx[b, 0] >= 0]
        np.testing.assert_array_equal(live, np.arange(c + 1))


def test_decode_ignores_rows_past_p():
    """Cache rows after p (here NaN) never reach the output or the selection."""
    rng = np.random.default_rng(22)
    blk, Hq, Hkv, D, Tmax, p = 8, 4, 2, 8, 200, 133
    q = rng.standard_normal((1, Hq, D))
    k, v = rng.standard_normal((1, Tmax, Hkv, D)), rng.standard_normal((1, Tmax, Hkv, D))
    y0, i0, _ = oracle.sparse_decode(q, k, v, [p], blk=blk, topk=3)
    k[:, p + 1:] = np.nan
    v[:, p + 1:] = np.nan
    y1, i1, _ = oracle.sparse_decode(q, k, v, [p], blk=blk, topk=3)
    np.testing.assert_array_equal(i0, i1)
    np.testing.assert_array_equal(y0, y1)
    assert np.all(np.isfinite(y1))


def test_decode_selection_bruteforce():
    """The decode selection is the brute-force top-k of the block-mean scores over the
    candidates n_init <= j <= c - n_local, united with the init and local blocks."""
    rng = np.random.default_rng(23)
    blk, Hq, Hkv, D, Tmax = 4, 4, 2, 6, 160
    q = rng.standard_normal((4, Hq, D))
    k, v = rng.standard_normal((4, Tmax, Hkv, D)), rng.standard_normal((4, Tmax, Hkv, D))
    pos = [159, 100, 63, 17]
    topk, n_init, n_local = 5, 1, 2
    _, idx, _ = oracle.sparse_decode(q, k, v, pos, blk=blk, topk=topk, n_init=n_init,
                                     n_local=n_local)
    G = Hq // Hkv
    for b, p in enumerate(pos):
        c = p // blk
        for hk in range(Hkv):
            qs = q[b, hk * G:(hk + 1) * G].sum(0)
            cand = list(range(n_init, c - n_local + 1))
            score = {j: qs @ k[b, j * blk:(j + 1) * blk, hk].mean(0) for j in cand}
            best = sorted(cand, key=lambda j: (-score[j], j))[:topk]
            want = sorted(set(range(min(n_init, c + 1))) | set(best) |
                          set(range(max(n_init, c - n_local + 1), c + 1)))
            got = idx[b, hk][idx[b, hk] >= 0].tolist()
            assert got == want, (b, hk)


# ---------------------------------------------------------------- per-head softmax selection
def test_head_softmax_scores_sum_to_group_size():
    """Each head's softmax over a row's candidates sums to 1, so a row's scores sum to
    the number of heads in the group (a wrong normalisation axis breaks this)."""
    rng = np.random.default_rng(21)
    blk, D, Hq, Hkv = 8, 16, 8, 2
    T = blk * 40 + 5
    q, k = rng.standard_normal((1, T, Hq, D)), rng.standard_normal((1, T, Hkv, D))
    rows = [blk * 5, blk * 17 + 3, T - 1]
    _, _, sc = oracle.sparse_select(q[:, rows], k, blk=blk, topk=4, rows=rows, want_scores=True,
                                    score="head_softmax")
    for r in range(len(rows)):
        for hk in range(Hkv):
            assert np.isclose(np.nansum(sc[0, hk, r]), Hq // Hkv, rtol=1e-12)


def test_head_softmax_one_head_is_softmax_of_group_scores():
    """With one query head per KV head the score is the softmax (scipy) of the
    group-sum score over the row's candidates, and the choice is the same."""
    from scipy.special import softmax

    rng = np.random.default_rng(22)
    blk, D, H = 8, 16, 3
    T = blk * 30 + 7
    q, k = rng.standard_normal((1, T, H, D)), rng.standard_normal((1, T, H, D))
    rows = list(range(blk * 3, T, 13))
    i0, _, s0 = oracle.sparse_select(q[:, rows], k, blk=blk, topk=5, rows=rows, want_scores=True)
    i1, _, s1 = oracle.sparse_select(q[:, rows], k, blk=blk, topk=5, rows=rows, want_scores=True,
                                     score="head_softmax")
    for hk in range(H):
        for r in range(len(rows)):
            m = ~np.isnan(s0[0, hk, r])
            if m.any():
                assert np.allclose(s1[0, hk, r][m], softmax(s0[0, hk, r][m]), rtol=1e-12,
                                   atol=1e-15)
    assert np.array_equal(i0, i1)


def test_head_softmax_planted_closed_form():
    """Every candidate block's keys are zero except block J, whose keys all equal u, and
    query head h is alpha_h * u: s_{h,J} = a_h = alpha_h |u|^2 / sqrt(D), 0 elsewhere, so
    score_J = sum_h e^{a_h} / (e^{a_h} + n - 1) and every other candidate scores
    sum_h 1 / (e^{a_h} + n - 1) (n candidates)."""
    blk, D, Hq = 8, 8, 4
    nb = 14
    T = blk * nb
    u = RNG.standard_normal(D) * 0.5
    alpha = np.array([0.3, -0.7, 1.1, 0.05])
    J = 6
    k = np.zeros((1, T, 1, D))
    k[0, J * blk:(J + 1) * blk, 0] = u
    q = np.zeros((1, T, Hq, D))
    for h in range(Hq):
        q[0, :, h] = alpha[h] * u
    t = T - 1
    _, _, sc = oracle.sparse_select(q[:, [t]], k, blk=blk, topk=3, rows=[t], want_scores=True,
                                    score="head_softmax")
    c = t // blk
    n = c - 2  # candidates 1 .. c - 2
    a = alpha * (u @ u) / math.sqrt(D)
    want_J = np.sum(np.exp(a) / (np.exp(a) + n - 1))
    want_other = np.sum(1.0 / (np.exp(a) + n - 1))
    row = sc[0, 0, 0]
    assert np.isclose(row[J - 1], want_J, rtol=1e-12)
    for j in range(1, c - 1):
        if j != J:
            assert np.isclose(row[j - 1], want_other, rtol=1e-12)


# ----------------------------------------------------------------------------
# Input projection of a Lightning layer with its preparation, and the recurrence on
# prepared operands (the fused hybrid-layer epilogue)
# ----------------------------------------------------------------------------

def test_matmul_nt_matches_numpy():
    """y = x W^T against numpy's matrix product (a transposed operand would fail)."""
    rng = np.random.default_rng(71)
    x, w = rng.standard_normal((37, 96)), rng.standard_normal((80, 96))
    np.testing.assert_allclose(oracle.matmul_nt(x, w), x @ w.T, rtol=1e-12, atol=1e-12)


def _proj_case(B=2, T=9, hidden=48, H=3, D=8, seed=72):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, T, hidden))
    w = rng.standard_normal((4 * H * D, hidden)) / math.sqrt(hidden)
    return x, w


def test_projection_sections_v_and_gate():
    """v is the third block of W's rows applied to x, gate = expit(fourth block)
    (scipy's logistic function), each head taking D consecutive rows."""
    from scipy.special import expit
    B, T, hidden, H, D = 2, 9, 48, 3, 8
    x, w = _proj_case(B, T, hidden, H, D)
    qh, kh, v, gate = oracle.lightning_projection(x, w, H=H, D=D, pos0=5)
    y = (x.reshape(-1, hidden) @ w.T).reshape(B, T, 4, H, D)
    np.testing.assert_allclose(v, y[:, :, 2], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gate, expit(y[:, :, 3]), rtol=1e-12, atol=1e-15)


def test_projection_qk_at_position_zero_is_rmsnorm():
    """At position 0 (pos0 = 0, token 0) the rotation is the identity: qh, kh are the
    projected q, k divided by their RMS (times the norm weight)."""
    B, T, hidden, H, D = 1, 4, 48, 3, 8
    x, w = _proj_case(B, T, hidden, H, D, seed=73)
    rng = np.random.default_rng(74)
    qw, kw = 1 + 0.1 * rng.standard_normal(D), 1 + 0.1 * rng.standard_normal(D)
    qh, kh, _, _ = oracle.lightning_projection(x, w, qw, kw, H=H, D=D, pos0=0, eps=1e-6)
    y = (x.reshape(-1, hidden) @ w.T).reshape(B, T, 4, H, D)
    for sec, out, wt in ((0, qh, qw), (1, kh, kw)):
        raw = y[0, 0, sec]
        want = raw / np.sqrt(np.mean(raw * raw, axis=-1, keepdims=True) + 1e-6) * wt
        np.testing.assert_allclose(out[0, 0], want, rtol=1e-12)


def test_projection_rope_relative_and_norm_preserving():
    """For the same hidden state placed at two positions, qh has the same norm (RoPE is
    a rotation) and qh(m) . kh(n) depends only on m - n."""
    B, T, hidden, H, D = 1, 1, 48, 1, 8
    x, w = _proj_case(B, T, hidden, H, D, seed=75)
    prep = {p: oracle.lightning_projection(x, w, H=H, D=D, pos0=p) for p in (3, 10, 103, 110)}
    q3, k10 = prep[3][0][0, 0, 0], prep[10][1][0, 0, 0]
    q103, k110 = prep[103][0][0, 0, 0], prep[110][1][0, 0, 0]
    assert np.isclose(q3 @ k10, q103 @ k110, rtol=1e-10)
    assert np.isclose(np.linalg.norm(q3), np.linalg.norm(q103), rtol=1e-12)
    assert not np.isclose(q3 @ k10, prep[3][0][0, 0, 0] @ prep[103][1][0, 0, 0], rtol=1e-3)


def test_projection_positions_follow_the_token_index():
    """Token t of each sequence sits at pos0 + t (the batch index does not shift it)."""
    B, T, hidden, H, D = 2, 5, 48, 2, 8
    x, w = _proj_case(B, T, hidden, H, D, seed=76)
    x[1] = x[0]
    qh, kh, _, _ = oracle.lightning_projection(x, w, H=H, D=D, pos0=7)
    np.testing.assert_allclose(qh[1], qh[0], rtol=1e-13)
    one, _, _, _ = oracle.lightning_projection(x[:, 3:4], w, H=H, D=D, pos0=10)
    np.testing.assert_allclose(one[:, 0], qh[:, 3], rtol=1e-12)


def test_prepared_recurrence_equals_raw_recurrence():
    """Fed the prepared operands of the raw q, k (qk_prep at each position) and
    sigmoid(g), the prepared recurrence gives the raw recurrence's outputs and state."""
    rng = np.random.default_rng(77)
    B, T, H, D = 2, 11, 2, 8
    q, k, v, g = (rng.standard_normal((B, T, H, D)) for _ in range(4))
    S0 = 0.1 * rng.standard_normal((B, H, D, D))
    y_raw, S_raw = oracle.lightning_recurrent(q, k, v, g, S0, pos0=4)
    qh = np.empty_like(q)
    kh = np.empty_like(k)
    for b in range(B):
        for t in range(T):
            for h in range(H):
                qh[b, t, h] = oracle.qk_prep(q[b, t, h], pos=4 + t)
                kh[b, t, h] = oracle.qk_prep(k[b, t, h], pos=4 + t)
    y, S = oracle.lightning_recurrent_prepared(qh, kh, v, 1 / (1 + np.exp(-g)), S0)
    np.testing.assert_allclose(y, y_raw, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, S_raw, rtol=1e-12, atol=1e-12)


def test_prepared_recurrence_quadratic_form():
    """Unrolled: y_t = gate_t * (qh_t^T S0 + sum_{s<=t} (qh_t . kh_s) v_s), by numpy."""
    rng = np.random.default_rng(78)
    B, T, H, D = 1, 13, 2, 8
    qh, kh, v, gate = (rng.standard_normal((B, T, H, D)) for _ in range(4))
    S0 = rng.standard_normal((B, H, D, D))
    y, S = oracle.lightning_recurrent_prepared(qh, kh, v, gate, S0)
    for h in range(H):
        P = np.tril(qh[0, :, h] @ kh[0, :, h].T)
        want = (P @ v[0, :, h] + qh[0, :, h] @ S0[0, h]) * gate[0, :, h]
        np.testing.assert_allclose(y[0, :, h], want, rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(S[0, h], S0[0, h] + kh[0, :, h].T @ v[0, :, h], rtol=1e-12)
