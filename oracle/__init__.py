"""fp64 CPU oracle for the SALA hybrid-attention hot path.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  The product
path (the CUDA library and its binding) never imports, links or calls it, and
this package imports nothing from the product.

The arithmetic lives in ``sala_oracle.c`` (plain loops in double precision);
this module compiles it with gcc and marshals numpy arrays.  Every function
takes and returns contiguous float64 arrays in [B, rows, heads, D] layout.

Pins: every routine here is pinned by the CPU tests in ``tests/test_oracle_pins.py``
against closed forms, invariants, brute force or library routines (see the test
docstrings).  Nothing here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sala_oracle.c")
_LIB = os.path.join(_HERE, "libsala_oracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i32p = ctypes.POINTER(ctypes.c_int32)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math) if stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i, d, i64 = ctypes.c_int, ctypes.c_double, ctypes.c_int64
        lib.oracle_qk_prep.argtypes = [_dp, _dp, i, d, d, d, _dp]
        lib.oracle_lightning_recurrent.argtypes = [
            _dp, _dp, _dp, _dp, _dp, _dp, _dp, i, i, i, i, i64, d, d, _i64p, i, _dp, _dp]
        lib.oracle_lightning_quadratic.argtypes = [
            _dp, _dp, _dp, _dp, _dp, _dp, _dp, i, i, i, i, i64, d, d, _dp]
        lib.oracle_lightning_chunked.argtypes = [
            _dp, _dp, _dp, _dp, _dp, _dp, _dp, i, i, i, i, i64, d, d, i, _dp, _dp]
        lib.oracle_lightning_decode.argtypes = [
            _dp, _dp, _dp, _dp, _dp, _dp, _dp, _i64p, i, i, i, d, d, _dp]
        lib.oracle_block_means.argtypes = [_dp, i, i, i, i, i, _dp]
        lib.oracle_sparse_select.argtypes = [
            _dp, _dp, i, i, i, i, i, i, i, i, i, _i64p, i, _i32p, _dp, _dp, i]
        lib.oracle_sparse_select_mode.argtypes = [
            _dp, _dp, i, i, i, i, i, i, i, i, i, _i64p, i, _i32p, _dp, _dp, i, i]
        lib.oracle_attention.argtypes = [
            _dp, _dp, _dp, _dp, _i32p, i, i, i, i, i, i, i, d, _i64p, i, _dp]
        lib.oracle_lightning_recurrent_prepared.argtypes = [
            _dp, _dp, _dp, _dp, _dp, i, i, i, i, _dp, _dp]
        lib.oracle_matmul_nt.argtypes = [_dp, _dp, i64, i, i, _dp]
        lib.oracle_lightning_projection.argtypes = [
            _dp, _dp, _dp, _dp, i, i, i, i, i, i64, d, d, _dp, _dp, _dp, _dp]
        for f in ("oracle_qk_prep", "oracle_lightning_recurrent", "oracle_lightning_quadratic",
                  "oracle_lightning_chunked", "oracle_lightning_decode", "oracle_block_means",
                  "oracle_sparse_select", "oracle_sparse_select_mode", "oracle_attention",
                  "oracle_lightning_recurrent_prepared", "oracle_matmul_nt",
                  "oracle_lightning_projection"):
            getattr(lib, f).restype = None
        _lib = lib
    return _lib


def _d(a):
    """Contiguous float64 view (or None) and its pointer."""
    if a is None:
        return None, None
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    return a, a.ctypes.data_as(_dp)


def _rows(rows, T):
    if rows is None:
        return None, None, T
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    if r.ndim != 1 or (r.size and (np.any(np.diff(r) <= 0) or r[0] < 0 or r[-1] >= T)):
        raise ValueError("rows must be strictly ascending positions in [0, T)")
    return r, r.ctypes.data_as(_i64p), int(r.size)


def qk_prep(x, w=None, *, eps=1e-6, pos=0, base=10000.0):
    """RMSNorm over the last axis (optional weight) then rotate-half RoPE at `pos`."""
    lib = _load()
    x, xp = _d(x)
    w, wp = _d(w)
    y = np.empty_like(x)
    lib.oracle_qk_prep(xp, wp, x.shape[-1], eps, float(pos), base, y.ctypes.data_as(_dp))
    return y


def lightning_recurrent(q, k, v, g=None, S0=None, qw=None, kw=None, *, pos0=0,
                        base=10000.0, eps=1e-6, rows: Optional[Sequence[int]] = None):
    """Recurrent Lightning attention.  q,k,v,g: [B,T,H,D].  Returns (y, S_final);
    y is [B, len(rows), H, D] when rows are given, else [B,T,H,D]."""
    lib = _load()
    B, T, H, D = np.shape(q)
    (q, qp), (k, kp), (v, vp), (g, gp) = _d(q), _d(k), _d(v), _d(g)
    (S0, sp), (qw, qwp), (kw, kwp) = _d(S0), _d(qw), _d(kw)
    r, rp, nrows = _rows(rows, T)
    y = np.zeros((B, nrows, H, D))
    S = np.zeros((B, H, D, D))
    lib.oracle_lightning_recurrent(qp, kp, vp, gp, sp, qwp, kwp, B, T, H, D, int(pos0), base, eps,
                                   rp, nrows, y.ctypes.data_as(_dp), S.ctypes.data_as(_dp))
    return y, S


def lightning_recurrent_prepared(qh, kh, v, gate=None, S0=None):
    """Recurrent Lightning attention on prepared operands: qh, kh already normalised and
    rotated, `gate` the output multiplier (sigmoid already applied) or None.
    qh, kh, v, gate: [B,T,H,D].  Returns (y [B,T,H,D], S_final)."""
    lib = _load()
    B, T, H, D = np.shape(qh)
    (qh, qp), (kh, kp), (v, vp), (gate, gp), (S0, sp) = _d(qh), _d(kh), _d(v), _d(gate), _d(S0)
    y = np.zeros((B, T, H, D))
    S = np.zeros((B, H, D, D))
    lib.oracle_lightning_recurrent_prepared(qp, kp, vp, gp, sp, B, T, H, D,
                                            y.ctypes.data_as(_dp), S.ctypes.data_as(_dp))
    return y, S


def matmul_nt(x, w):
    """y = x W^T for x [M, K], W [N, K] (plain fp64 loops)."""
    lib = _load()
    (x, xp), (w, wp) = _d(x), _d(w)
    M, K = x.shape
    N = w.shape[0]
    y = np.zeros((M, N))
    lib.oracle_matmul_nt(xp, wp, M, K, N, y.ctypes.data_as(_dp))
    return y


def lightning_projection(x, w, qw=None, kw=None, *, H, D, pos0=0, base=10000.0, eps=1e-6):
    """Lightning-layer inputs from hidden states x [B,T,hidden] and the projection weight
    W [4 H D, hidden] (rows: q heads, then k, v, g heads).  Returns (qh, kh, v, gate),
    each [B,T,H,D]: q, k normalised and rotated at pos0 + t, v as projected, gate =
    sigmoid(g)."""
    lib = _load()
    B, T, hidden = np.shape(x)
    (x, xp), (w, wp), (qw, qwp), (kw, kwp) = _d(x), _d(w), _d(qw), _d(kw)
    if w.shape != (4 * H * D, hidden):
        raise ValueError("W must be [4 H D, hidden]")
    outs = [np.zeros((B, T, H, D)) for _ in range(4)]
    lib.oracle_lightning_projection(xp, wp, qwp, kwp, B, T, hidden, H, D, int(pos0), base, eps,
                                    *(o.ctypes.data_as(_dp) for o in outs))
    return tuple(outs)


def lightning_quadratic(q, k, v, g=None, S0=None, qw=None, kw=None, *, pos0=0,
                        base=10000.0, eps=1e-6):
    """Quadratic masked form of the same attention; returns y [B,T,H,D]."""
    lib = _load()
    B, T, H, D = np.shape(q)
    (q, qp), (k, kp), (v, vp), (g, gp) = _d(q), _d(k), _d(v), _d(g)
    (S0, sp), (qw, qwp), (kw, kwp) = _d(S0), _d(qw), _d(kw)
    y = np.zeros((B, T, H, D))
    lib.oracle_lightning_quadratic(qp, kp, vp, gp, sp, qwp, kwp, B, T, H, D, int(pos0), base, eps,
                                   y.ctypes.data_as(_dp))
    return y


def lightning_chunked(q, k, v, g=None, S0=None, qw=None, kw=None, *, chunk, pos0=0,
                      base=10000.0, eps=1e-6):
    """Chunked form with chunk length `chunk`; returns (y, S_final)."""
    lib = _load()
    B, T, H, D = np.shape(q)
    (q, qp), (k, kp), (v, vp), (g, gp) = _d(q), _d(k), _d(v), _d(g)
    (S0, sp), (qw, qwp), (kw, kwp) = _d(S0), _d(qw), _d(kw)
    y = np.zeros((B, T, H, D))
    S = np.zeros((B, H, D, D))
    lib.oracle_lightning_chunked(qp, kp, vp, gp, sp, qwp, kwp, B, T, H, D, int(pos0), base, eps,
                                 int(chunk), y.ctypes.data_as(_dp), S.ctypes.data_as(_dp))
    return y, S


def lightning_decode(q, k, v, g, S, pos, qw=None, kw=None, *, base=10000.0, eps=1e-6,
                     inplace=False):
    """One decode step.  q,k,v,g: [B,H,D]; S: [B,H,D,D]; pos: [B].
    Returns (y [B,H,D], S_new).  With inplace=True and S a C-contiguous float64 array,
    S itself is updated (and returned) instead of a copy."""
    lib = _load()
    B, H, D = np.shape(q)
    (q, qp), (k, kp), (v, vp), (g, gp) = _d(q), _d(k), _d(v), _d(g)
    (qw, qwp), (kw, kwp) = _d(qw), _d(kw)
    if not (inplace and isinstance(S, np.ndarray) and S.dtype == np.float64
            and S.flags.c_contiguous):
        S = np.array(S, dtype=np.float64, copy=True, order="C")
    p = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    y = np.zeros((B, H, D))
    lib.oracle_lightning_decode(qp, kp, vp, gp, S.ctypes.data_as(_dp), qwp, kwp,
                                p.ctypes.data_as(_i64p), B, H, D, base, eps, y.ctypes.data_as(_dp))
    return y, S


def block_means(k, blk=64):
    """Mean of each complete block of keys: [B, T//blk, Hkv, D]."""
    lib = _load()
    B, T, Hkv, D = np.shape(k)
    k, kp = _d(k)
    out = np.zeros((B, T // blk, Hkv, D))
    lib.oracle_block_means(kp, B, T, Hkv, D, blk, out.ctypes.data_as(_dp))
    return out


SCORE_MODES = {"group_sum": 0, "head_softmax": 1}


def sparse_select(q, k, *, blk=64, topk=64, n_init=1, n_local=2, rows=None, T=None,
                  want_scores=False, score="group_sum"):
    """Block selection.  q: [B, nrows, Hq, D] (rows listed in `rows`, else all T);
    k: [B, T, Hkv, D].  Returns (idx [B,Hkv,nrows,n_sel] int32, gap [B,Hkv,nrows])
    and, with want_scores, candidate scores [B,Hkv,nrows,max_cand] (NaN = none).
    score="group_sum": (1/sqrt(D)) sum over the group's heads of q_h . Kbar_j;
    score="head_softmax": each head's scaled dot products softmax-normalised over the
    row's candidates, then summed over the group's heads."""
    if score not in SCORE_MODES:
        raise ValueError(f"score must be one of {sorted(SCORE_MODES)}")
    lib = _load()
    B, nr, Hq, D = np.shape(q)
    _, Tk, Hkv, _ = np.shape(k)
    T = Tk if T is None else T
    (q, qp), (k, kp) = _d(q), _d(k)
    r, rp, nrows = _rows(rows, T)
    if nrows != nr:
        raise ValueError("q rows do not match `rows`")
    n_sel = n_init + topk + n_local
    idx = np.zeros((B, Hkv, nrows, n_sel), dtype=np.int32)
    gap = np.zeros((B, Hkv, nrows))
    max_cand = max(1, T // blk)
    sc = np.zeros((B, Hkv, nrows, max_cand)) if want_scores else None
    lib.oracle_sparse_select_mode(qp, kp, B, T, Hq, Hkv, D, blk, topk, n_init, n_local, rp,
                                  nrows, idx.ctypes.data_as(_i32p), gap.ctypes.data_as(_dp),
                                  sc.ctypes.data_as(_dp) if sc is not None else None, max_cand,
                                  SCORE_MODES[score])
    return (idx, gap, sc) if want_scores else (idx, gap)


def attention(q, k, v, g=None, idx=None, *, blk=64, scale=None, rows=None):
    """Softmax attention over selected blocks (idx [B,Hkv,nrows,n_sel]) or, with
    idx=None, dense causal attention.  q,g: [B,nrows,Hq,D]; k,v: [B,T,Hkv,D]."""
    lib = _load()
    B, nr, Hq, D = np.shape(q)
    _, T, Hkv, _ = np.shape(k)
    (q, qp), (k, kp), (v, vp), (g, gp) = _d(q), _d(k), _d(v), _d(g)
    r, rp, nrows = _rows(rows, T)
    if nrows != nr:
        raise ValueError("q rows do not match `rows`")
    if idx is not None:
        idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
        n_sel = idx.shape[-1]
        ip = idx.ctypes.data_as(_i32p)
    else:
        n_sel, ip = 0, None
    sc = 1.0 / np.sqrt(D) if scale is None else float(scale)
    y = np.zeros((B, nrows, Hq, D))
    lib.oracle_attention(qp, kp, vp, gp, ip, n_sel, B, T, Hq, Hkv, D, blk, sc, rp, nrows,
                         y.ctypes.data_as(_dp))
    return y


def sparse_decode(q, k_cache, v_cache, pos, g=None, *, blk=64, topk=64, n_init=1, n_local=2,
                  scale=None, want_scores=False):
    """Sparse-layer decode step: for each sequence b, row p = pos[b] of the prefill
    computation (sparse_select then attention) over cache rows 0..p only.
    q, g: [B, Hq, D]; k_cache, v_cache: [B, Tmax, Hkv, D]; pos: [B] ints.
    Returns (y [B, Hq, D], idx [B, Hkv, n_sel] int32, gap [B, Hkv]) and, with
    want_scores, the candidate scores [B, Hkv, Tmax // blk] (NaN = not a candidate)."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, D = q.shape
    Hkv = np.shape(k_cache)[2]
    n_sel = n_init + topk + n_local
    y = np.zeros((B, Hq, D))
    idx = np.zeros((B, Hkv, n_sel), dtype=np.int32)
    gap = np.zeros((B, Hkv))
    ncap = max(1, np.shape(k_cache)[1] // blk)
    sc = np.full((B, Hkv, ncap), np.nan)
    for b in range(B):
        p = int(pos[b])
        kk = np.asarray(k_cache[b:b + 1, :p + 1], dtype=np.float64)
        vv = np.asarray(v_cache[b:b + 1, :p + 1], dtype=np.float64)
        qr = q[b][None, None]
        gr = None if g is None else np.asarray(g[b], dtype=np.float64)[None, None]
        ib, gb, sb = sparse_select(qr, kk, blk=blk, topk=topk, n_init=n_init, n_local=n_local,
                                   rows=[p], T=p + 1, want_scores=True)
        y[b] = attention(qr, kk, vv, gr, idx=ib, blk=blk, scale=scale, rows=[p])[0, 0]
        idx[b] = ib[0, :, 0]
        gap[b] = gb[0, :, 0]
        sc[b, :, :sb.shape[-1]] = sb[0, :, 0]
    return (y, idx, gap, sc) if want_scores else (y, idx, gap)
