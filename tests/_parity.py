"""Shared helpers for the GPU parity tests: tolerance metric and index-set checks.

Tolerances (outputs and states): max|err| / rms(ref) <= 1e-2 for bf16 inputs and
<= 1e-5 for fp32 inputs.  For bf16 OUTPUTS the kernel's last step is a
round-to-nearest-even into bf16, which alone moves a value by up to half a
bf16 ulp (2^-8 relative); the bound is applied to the value before that final
rounding, i.e. each element's error is reduced by half an ulp of the stored
output before the maximum is taken.  fp32 outputs and the fp32 state get no
allowance.
"""
import numpy as np

TOL_BF16 = 1e-2
TOL_F32 = 1e-5
GAP_TIE = 1e-4


def rel_err(out, ref, bf16_out: bool) -> float:
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(out - ref)
    if bf16_out:
        e = np.floor(np.log2(np.maximum(np.abs(out), 1e-30)))
        err = np.maximum(err - np.exp2(e - 8), 0.0)
    rms = np.sqrt(np.mean(ref * ref))
    return float(err.max() / rms) if rms > 0 else float(err.max())


def rel_err_bf16_pair(a, b) -> float:
    """Same 1e-2 rule for two bf16 OUTPUTS of the library (no fp64 reference):
    each side was rounded to bf16 once, so half an ulp of each is allowed."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    def half_ulp(x):
        return np.exp2(np.floor(np.log2(np.maximum(np.abs(x), 1e-30))) - 8)
    err = np.maximum(np.abs(a - b) - half_ulp(a) - half_ulp(b), 0.0)
    rms = np.sqrt(np.mean(b * b))
    return float(err.max() / rms) if rms > 0 else float(err.max())


def raw_rel_err(out, ref) -> float:
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(out - ref).max() / max(np.sqrt(np.mean(ref * ref)), 1e-300))


def check_index_sets(idx_gpu, idx_ref, gap, scores, t, *, topk, n_init=1, n_local=2, blk=64,
                     tie_band=None):
    """Selected block sets against the oracle's.

    idx_gpu, idx_ref: [..., n_sel] (ascending, -1 padded); gap: [...] the oracle's
    topk-th minus (topk+1)-th candidate score; scores: [..., max_cand] the oracle's
    candidate scores by block offset j - n_init (NaN where j is not a candidate);
    t: each row's query position, broadcast against `gap`.

    Rows must be bit-exact, except rows whose gap is below the tie band (1e-4, or
    `tie_band`, a scalar or an array shaped like `gap`).  Such a row may differ from
    the oracle's only by near-tied candidates, and must still be a valid selection:
      * same number of entries, strictly ascending, every entry in [0, c] (c = t // blk);
      * every forced block present: init blocks [0, n_init) and the local window
        [c - n_local + 1, c], both clipped to [0, c];
      * every block in the symmetric difference is a candidate (n_init <= j <= c - n_local)
        whose oracle score lies within the band of the oracle's topk-th score.
    Returns (rows that differ, rows checked)."""
    idx_gpu = np.asarray(idx_gpu)
    idx_ref = np.asarray(idx_ref)
    gap = np.asarray(gap, dtype=np.float64)
    scores = np.asarray(scores, dtype=np.float64)
    t = np.broadcast_to(np.asarray(t, dtype=np.int64), gap.shape)
    band = np.broadcast_to(np.asarray(GAP_TIE if tie_band is None else tie_band,
                                      dtype=np.float64), gap.shape)
    same = (idx_gpu == idx_ref).all(axis=-1)
    tie = gap < band
    bad = ~same & ~tie
    assert not bad.any(), f"{int(bad.sum())} rows differ without a near-tie"
    for r in np.argwhere(~same):
        r = tuple(r)
        a, b = idx_gpu[r], idx_ref[r]
        va, vb = a[a >= 0], b[b >= 0]
        c = int(t[r]) // blk
        assert len(va) == len(vb), (r, va, vb)
        assert np.all(np.diff(va) > 0), (r, va)
        assert va.size == 0 or (va[0] >= 0 and va[-1] <= c), (r, va, c)
        assert np.all(a[len(va):] == -1), (r, a)
        forced = set(range(0, min(n_init, c + 1))) | set(range(max(0, c - n_local + 1), c + 1))
        assert forced <= set(va.tolist()), (r, sorted(forced - set(va.tolist())))
        sc = scores[r]
        cand = np.where(np.isnan(sc), -np.inf, sc)
        kth = -np.sort(-cand)[topk - 1]
        for j in set(va.tolist()) ^ set(vb.tolist()):
            assert n_init <= j <= c - n_local, (r, j, "not a candidate")
            assert abs(sc[j - n_init] - kth) <= band[r], (r, j, sc[j - n_init], kth)
    return int((~same).sum()), int(same.size)
