"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and host-side argument validation rejects bad calls before
any launch."""
import ctypes
import os
import re

import pytest

import sparse_attention_long_lightning_b200 as sala
from sparse_attention_long_lightning_b200 import build as sala_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sala.h")


@pytest.fixture(scope="module")
def lib():
    sala_build.build()
    return sala.load_library()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sala_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_four_operations():
    names = declared_symbols()
    for fn in ("sala_lightning_prefill", "sala_lightning_decode", "sala_sparse_select",
               "sala_sparse_attn"):
        assert fn in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert sala.status_string(0) == "SALA_OK"
    assert sala.status_string(1) == "SALA_ERR_INVALID_ARG"
    assert sala.status_string(6) == "SALA_ERR_RANGE"
    assert sala.status_string(7) == "SALA_ERR_BOUNDS"
    assert "sm_100a" in sala.version() and "SALA_DEBUG" not in sala.version()
    # the release library has no device index checks
    assert sala.debug_bounds_line() == -1


def test_debug_library_exports_every_declared_symbol():
    """libsala_debug.so (SALA_DEBUG: device index checks) is the same ABI."""
    path = sala_build.build(debug=True)
    dbg = ctypes.CDLL(path)
    for name in declared_symbols():
        assert hasattr(dbg, name), name
    dbg.sala_version.restype = ctypes.c_char_p
    assert b"SALA_DEBUG" in dbg.sala_version()


Z = sala.SalaStrides(0, 0, 0)


def _prefill(lib, q=None, D=128, chunk=128, dt=1, T=16, B=1, H=1, base=10000.0, pos0=0):
    p = ctypes.c_void_p(16) if q is None else q
    st = sala.SalaStrides(T * H * D, H * D, D)
    return lib.sala_lightning_prefill(p, p, p, None, p, p, None, None, B, T, H, D, st, st, st, Z,
                                      st, chunk, pos0, base, 1e-6, 1, None, 0, dt, None)


def test_prefill_rejects_bad_arguments(lib):
    assert _prefill(lib, q=ctypes.c_void_p(0)) == 1          # null pointer
    assert _prefill(lib, q=ctypes.c_void_p(8)) == 1          # misaligned
    assert _prefill(lib, D=96) == 2                          # unsupported head dim
    assert _prefill(lib, chunk=32) == 2                      # unsupported chunk
    assert _prefill(lib, dt=7) == 2                          # unknown dtype
    assert _prefill(lib, B=0) == 1
    assert _prefill(lib, T=-1) == 1
    assert _prefill(lib, base=1.0) == 1
    assert _prefill(lib, pos0=-3) == 1
    p = ctypes.c_void_p(16)
    bad = sala.SalaStrides(1, 1, 1)                          # rows not 16-byte aligned
    assert lib.sala_lightning_prefill(p, p, p, None, p, p, None, None, 1, 4, 1, 128, bad, bad,
                                      bad, Z, bad, 128, 0, 10000.0, 1e-6, 1, None, 0, 1,
                                      None) == 1


def test_decode_rejects_bad_arguments(lib):
    p = ctypes.c_void_p(16)
    st = sala.SalaStrides(128, 0, 128)
    assert lib.sala_lightning_decode(p, p, p, None, p, p, None, None, None, 1, 1, 128, st, st,
                                     st, Z, st, 10000.0, 1e-6, 1, None) == 1  # null pos
    assert lib.sala_lightning_decode(p, p, p, None, p, p, None, None, p, 1, 1, 48, st, st, st, Z,
                                     st, 10000.0, 1e-6, 1, None) == 2


def test_select_and_attn_reject_bad_arguments(lib):
    p = ctypes.c_void_p(16)
    st = sala.SalaStrides(64 * 2 * 128, 2 * 128, 128)
    # Hq not a multiple of Hkv
    assert lib.sala_sparse_select(p, p, 1, 64, 3, 2, 128, st, st, 64, 4, 1, 2, p, p, 1 << 20, 1,
                                  None) == 1
    # block size other than 64
    assert lib.sala_sparse_select(p, p, 1, 64, 2, 2, 128, st, st, 32, 4, 1, 2, p, p, 1 << 20, 1,
                                  None) == 2
    # workspace too small
    assert lib.sala_sparse_select(p, p, 1, 640, 2, 2, 128, st, st, 64, 4, 1, 2, p, p, 16, 1,
                                  None) == 5
    # fp32 sparse path is not provided
    assert lib.sala_sparse_attn(p, p, p, None, p, 67, p, 1, 64, 2, 2, 128, st, st, st, Z, st, 64,
                                0.0, p, 1 << 20, 0, None) == 2
    # group larger than one 16-row tile
    assert lib.sala_sparse_attn(p, p, p, None, p, 67, p, 1, 64, 64, 2, 128, st, st, st, Z, st, 64,
                                0.0, p, 1 << 20, 1, None) == 2
    # workspace too small for the fp16 copy of v
    assert lib.sala_sparse_attn(p, p, p, None, p, 67, p, 1, 64, 2, 2, 128, st, st, st, Z, st, 64,
                                0.0, p, 16, 1, None) == 5


def test_sparse_decode_rejects_bad_arguments(lib):
    p = ctypes.c_void_p(16)
    sq = sala.SalaStrides(32 * 128, 0, 128)
    sk = sala.SalaStrides(4096 * 2 * 128, 2 * 128, 128)

    def call(pos=p, Tmax=4096, Hq=32, Hkv=2, D=128, ws_bytes=1 << 26, dt=1, block=64):
        return lib.sala_sparse_decode(p, p, p, None, p, pos, p, None, 1, Tmax, Hq, Hkv, D, sq, sk,
                                      sk, Z, sq, block, 64, 1, 2, 0.0, p, ws_bytes, dt, None)
    assert call(pos=None) == 1                 # null pos
    assert call(Tmax=4000) == 1                # cache length not a multiple of 64
    assert call(Hq=33) == 1                    # Hq not a multiple of Hkv
    assert call(D=48) == 2                     # head_dim
    assert call(Hq=64) == 2                    # group of 32 heads > one 16-row tile
    assert call(block=32) == 2
    assert call(dt=0) == 2                     # fp32 not provided
    assert call(ws_bytes=16) == 5              # workspace too small
    # block means: kbar too short for the cache
    assert lib.sala_sparse_block_means(p, 1, 4096, 2, 128, sk, p, 63, 1, None) == 1
    assert lib.sala_sparse_block_means(p, 1, 4096, 2, 96, sk, p, 64, 1, None) == 2


def test_lightning_state_and_prefix_reject_bad_arguments(lib):
    p = ctypes.c_void_p(16)
    st = sala.SalaStrides(64 * 4 * 128, 4 * 128, 128)
    assert lib.sala_lightning_state(p, p, None, None, 1, 64, 4, 128, st, st, 128, 0, 10000.0,
                                    1e-6, 1, p, 1 << 24, 1, None) == 1  # null state
    assert lib.sala_lightning_state(p, p, p, None, 1, 64, 4, 48, st, st, 128, 0, 10000.0, 1e-6,
                                    1, p, 1 << 24, 1, None) == 2        # head_dim
    assert lib.sala_lightning_state(p, p, p, None, 1, 64, 4, 128, st, st, 128, -1, 10000.0,
                                    1e-6, 1, p, 1 << 24, 1, None) == 1  # negative position
    assert lib.sala_lightning_state(p, p, p, None, 1, 64, 4, 128, st, st, 128, 0, 10000.0, 1e-6,
                                    1, p, 16, 1, None) == 5             # workspace
    assert lib.sala_state_prefix_sum(p, 1024, 2, 512, p, 1, None) == 1  # overlapping sources
    assert lib.sala_state_prefix_sum(None, 1024, 2, 1024, p, 1, None) == 1
    assert lib.sala_state_prefix_sum(None, 1024, 0, 0, p, 1, None) == 0  # nothing to add


def test_sparse_decode_workspace_query():
    up = lambda x: (x + 255) // 256 * 256
    n = sala.sparse_decode_workspace(64, 131072, 32, 2, 128, 67)
    scores, idx, part = 64 * 2 * 2048 * 4, 64 * 2 * 67 * 4, 64 * 2 * 16 * 16 * 130 * 4
    assert n == up(scores) + up(idx) + up(part)
    assert sala.sparse_decode_workspace(1, 100, 32, 2, 128, 67) == 0


def test_workspace_queries(lib):
    nb = 131072 // 64
    means = nb * 2 * 128 * (4 + 2 + 2)                       # fp32 means + bf16 hi / lo
    # topk <= 64: block means only (scores and top-k fused)
    n = sala.sparse_select_workspace(1, 131072, 32, 2, 128, 64, 64)
    assert means <= n <= means + 1024
    # larger topk: plus a score scratch bounded by 1 GiB and the means' third bf16 part
    n = sala.sparse_select_workspace(1, 131072, 32, 2, 128, 64, 100)
    means3 = means + nb * 2 * 128 * 2
    assert means3 + (1 << 29) <= n <= means3 + (1 << 30) + 4096
    assert sala.sparse_select_workspace(1, 1 << 20, 32, 2, 128, 64, 200) <= (1 << 30) + (1 << 26)
    # fp16 copy of v, then 128 partial maxima and 128 partial sums of squares, one
    # exponent and one outlier flag per (sequence, KV head), each part 256-byte aligned
    assert sala.sparse_attn_workspace(1, 131072, 2, 128) == 131072 * 2 * 128 * 2 + 2 * 1024 + 2 * 256
    assert sala.sparse_attn_workspace(1, 0, 2, 128) == 0
    # Lightning (bf16, D128, chunk 128): segment states plus the segments' largest |v|
    n = sala.lightning_prefill_workspace(1, 131072, 32, 128, 128)
    G = n // (32 * 128 * 128 * 4)
    assert G >= 1 and n == 32 * G * 128 * 128 * 4 + 2 * ((32 * G * 4 + 255) // 256 * 256)


def test_head_softmax_select_rejects_bad_arguments(lib):
    p = ctypes.c_void_p(16)
    st = sala.SalaStrides(64 * 6 * 128, 6 * 128, 128)
    # group of 3 heads: not a power of two
    assert lib.sala_sparse_select_head_softmax(p, p, 1, 640, 6, 2, 128, st, st, 64, 4, 1, 2, p,
                                               p, 1 << 30, 1, None) == 2
    # Hq not a multiple of Hkv
    assert lib.sala_sparse_select_head_softmax(p, p, 1, 640, 3, 2, 128, st, st, 64, 4, 1, 2, p,
                                               p, 1 << 30, 1, None) == 1
    # workspace too small (the score scratch is always needed)
    need = sala.sparse_select_head_softmax_workspace(1, 640, 4, 2, 128)
    assert lib.sala_sparse_select_head_softmax(p, p, 1, 640, 4, 2, 128, st, st, 64, 4, 1, 2, p,
                                               p, need - 1, 1, None) == 5


def test_head_softmax_workspace_has_score_scratch():
    nb = 131072 // 64
    means = nb * 2 * 128 * (4 + 2 + 2)
    n = sala.sparse_select_head_softmax_workspace(1, 131072, 32, 2, 128)
    means3 = means + nb * 2 * 128 * 2  # hi / lo / lo2 bf16 parts of the means
    assert means3 + (1 << 29) <= n <= means3 + (1 << 30) + 4096
    assert n == sala.sparse_select_workspace(1, 131072, 32, 2, 128, 64, 100)
    assert sala.sparse_select_head_softmax_workspace(1, 0, 32, 2, 128) == 0


def test_row_window_calls_reject_bad_windows(lib):
    p = ctypes.c_void_p(16)
    st = sala.SalaStrides(64 * 2 * 128, 2 * 128, 128)
    ws = 1 << 30
    sel = lambda Tq, q0, Tk, score=0: lib.sala_sparse_select_rows(
        p, p, 1, Tq, q0, Tk, 2, 2, 128, st, st, 64, 4, 1, 2, score, p, p, ws, 1, None)
    att = lambda Tq, q0, Tk: lib.sala_sparse_attn_rows(
        p, p, p, None, p, 7, p, 1, Tq, q0, Tk, 2, 2, 128, st, st, st, Z, st, 64, 0.0, p, ws, 1,
        None)
    for fn in (sel, att):
        assert fn(64, 1, 64) == 1        # window runs past the keys
        assert fn(64, -1, 640) == 1      # negative first position
        assert fn(64, 0, 32) == 1        # fewer keys than query rows
        assert fn(0, 640, 640) == 0      # an empty window at the end is a no-op
    assert sel(64, 0, 640, score=2) == 1  # unknown score rule
    # the whole-sequence calls keep their own checks
    assert lib.sala_sparse_select_rows(p, p, 1, 64, 0, 64, 3, 2, 128, st, st, 64, 4, 1, 2, 0, p,
                                       p, ws, 1, None) == 1


def test_row_window_workspace_queries():
    nb = 131072 // 64
    means = nb * 2 * 128 * (4 + 2 + 2)
    # block means of all Tk keys; the score scratch (head softmax) sized by the Tq rows
    n = sala.sparse_select_rows_workspace(1, 16384, 131072, 32, 2, 128)
    assert n == sala.sparse_select_workspace(1, 131072, 32, 2, 128, 64, 64)
    assert means <= n <= means + 1024
    hs = sala.sparse_select_rows_workspace(1, 64, 131072, 32, 2, 128, score="head_softmax")
    assert hs == means + 2 * 64 * nb * 4 + nb * 2 * 128 * 2  # + the means' third part
    full = sala.sparse_select_rows_workspace(1, 131072, 131072, 32, 2, 128, score="head_softmax")
    assert full == sala.sparse_select_head_softmax_workspace(1, 131072, 32, 2, 128)
    assert sala.sparse_select_rows_workspace(1, 64, 0, 32, 2, 128) == 0


def test_tracing_wraps_compute_calls_only(lib):
    """With tracing on, compute entry points go through an NVTX range (and still return
    the library's status); workspace queries and status helpers are the bare calls."""
    raw = lib._cdll
    sala.set_tracing(True)
    try:
        traced = lib.sala_sparse_select
        assert traced is not raw.sala_sparse_select
        p = ctypes.c_void_p(16)
        st = sala.SalaStrides(64 * 2 * 128, 2 * 128, 128)
        assert traced(p, p, 1, 64, 3, 2, 128, st, st, 64, 4, 1, 2, p, p, 1 << 20, 1, None) == 1
        assert lib.sala_sparse_select_workspace is raw.sala_sparse_select_workspace
        assert lib.sala_status_string is raw.sala_status_string
    finally:
        sala.set_tracing(False)
    assert lib.sala_sparse_select is raw.sala_sparse_select
