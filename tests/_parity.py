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


def check_index_sets(idx_gpu, idx_ref, gap, tie_band=None):
    """Bit-exact per row, except rows whose oracle gap between the topk-th and
    (topk+1)-th candidate score is below the tie band (1e-4, or `tie_band`, a scalar
    or per-row array): there the chosen sets may differ only by near-tied members
    (same size, same forced blocks, every row sorted)."""
    idx_gpu = np.asarray(idx_gpu)
    idx_ref = np.asarray(idx_ref)
    same = (idx_gpu == idx_ref).all(axis=-1)
    tie = gap < (GAP_TIE if tie_band is None else tie_band)
    bad = ~same & ~tie
    assert not bad.any(), f"{int(bad.sum())} rows differ without a near-tie"
    # structural validity of the tied rows
    for r in np.argwhere(~same):
        a, b = idx_gpu[tuple(r)], idx_ref[tuple(r)]
        va, vb = a[a >= 0], b[b >= 0]
        assert len(va) == len(vb) and np.all(np.diff(va) > 0)
    return int((~same).sum()), int(same.size)
