"""CPU checks of the parity helpers themselves (no GPU): the index-set check must accept
the oracle's selection and valid near-tie alternatives, and reject selections with a
planted mistake (a forced block dropped, a block past the query's own, a non-tied
candidate swapped in, disorder, a wrong count)."""
import numpy as np
import pytest

import oracle
from sparse_attention_long_lightning_b200 import inputs
from tests._parity import check_index_sets, rel_err, rel_err_bf16_pair


def _case(seed=5, T=64 * 30 + 5, ties=False):
    s = inputs.sparse_inputs(1, T, 4, 1, 16, seed=seed)
    q = s.q.double().numpy()
    k = s.k.double().numpy()
    if ties:  # every block holds the same keys: all candidate scores of a row are equal
        k = np.tile(k[:, :64], (1, (T + 63) // 64, 1, 1))[:, :T]
    idx, gap, sc = oracle.sparse_select(q, k, topk=8, want_scores=True)
    return idx, gap, sc, np.arange(T)


def _fails(*a, **kw):
    with pytest.raises(AssertionError):
        check_index_sets(*a, **kw)


def test_accepts_oracle_and_tied_alternative():
    idx, gap, sc, t = _case(ties=True)
    check_index_sets(idx, idx, gap, sc, t, topk=8)
    # row t = 1500 (c = 23): every candidate is tied, so any 8 of them are valid
    r = (0, 0, 1500)
    alt = idx.copy()
    row = alt[r]
    chosen = set(row[row >= 0].tolist())
    cands = [j for j in range(1, 23 - 1) if j not in chosen]
    drop = [j for j in sorted(chosen) if 1 <= j <= 21][0]
    new = sorted((chosen - {drop}) | {cands[0]})
    alt[r][:len(new)] = new
    assert check_index_sets(alt, idx, gap, sc, t, topk=8)[0] == 1


def test_rejects_planted_mistakes():
    idx, gap, sc, t = _case(ties=True)
    r = (0, 0, 1500)  # c = 23; under exact ties the oracle takes {0, 1..8, 22, 23}
    assert idx[r][idx[r] >= 0].tolist() == [0, 1, 2, 3, 4, 5, 6, 7, 8, 22, 23]

    def planted(entries):
        bad = idx.copy()
        bad[r] = np.array(entries + [-1] * (idx.shape[-1] - len(entries)))
        return bad
    # a tied alternative (8 -> 9) is valid
    check_index_sets(planted([0, 1, 2, 3, 4, 5, 6, 7, 9, 22, 23]), idx, gap, sc, t, topk=8)
    # the init block replaced by a tied candidate
    _fails(planted([1, 2, 3, 4, 5, 6, 7, 8, 9, 22, 23]), idx, gap, sc, t, topk=8)
    # a local block replaced by a tied candidate
    _fails(planted([0, 1, 2, 3, 4, 5, 6, 7, 8, 9, 23]), idx, gap, sc, t, topk=8)
    # a block after the query's own block
    _fails(planted([0, 1, 2, 3, 4, 5, 6, 7, 22, 23, 24]), idx, gap, sc, t, topk=8)
    # one entry short
    _fails(planted([0, 1, 2, 3, 4, 5, 6, 7, 22, 23]), idx, gap, sc, t, topk=8)
    # out of order
    _fails(planted([0, 2, 1, 3, 4, 5, 6, 7, 8, 22, 23]), idx, gap, sc, t, topk=8)
    # a repeated entry
    _fails(planted([0, 1, 2, 3, 4, 5, 6, 7, 7, 22, 23]), idx, gap, sc, t, topk=8)


def test_rejects_non_tied_swap_and_accepts_tied_one():
    idx, gap, sc, t = _case(seed=6)
    # a late row with many candidates; give it a band just above its own gap
    r = (0, 0, 1800)
    c = 1800 // 64
    row_sc = sc[r]
    order = np.argsort(-np.where(np.isnan(row_sc), -np.inf, row_sc), kind="stable")
    kth_j, next_j, worst_j = order[7] + 1, order[8] + 1, order[c - 3] + 1
    band = np.zeros_like(gap)
    band[r] = gap[r] * 2 + 1e-12
    def swap(add):
        bad = idx.copy()
        v = sorted(set(bad[r][bad[r] >= 0].tolist()) - {kth_j} | {add})
        bad[r][:len(v)] = v
        return bad
    # the (topk+1)-th candidate is within the band of the topk-th: accepted
    assert check_index_sets(swap(next_j), idx, gap, sc, t, topk=8, tie_band=band)[0] == 1
    # the lowest-scoring candidate is not: rejected
    _fails(swap(worst_j), idx, gap, sc, t, topk=8, tie_band=band)
    # and without a near-tie the rows must match exactly
    _fails(swap(next_j), idx, gap, sc, t, topk=8)


def test_rel_err_allows_half_an_output_ulp_only():
    ref = np.array([1.0, -3.0, 0.5, 2.0])
    out = ref + np.array([0.0, 3.0 * 2.0 ** -9, 0.0, 0.0])  # half an ulp of -3 in bf16
    assert rel_err(out, ref, True) == 0.0
    assert rel_err(out, ref, False) > 0.0
    out2 = ref + np.array([0.0, 0.05, 0.0, 0.0])
    assert rel_err(out2, ref, True) > 0.01
    assert rel_err_bf16_pair(out2, ref) > 0.01
