"""B200-native SALA hybrid-attention hot path: thin Python binding over libsala.

Every call below marshals torch CUDA tensors into the C ABI of ``include/sala.h``
(pointers, sizes, element strides, the current CUDA stream) and raises
``SalaError`` on a non-zero status.  All arithmetic runs in the CUDA kernels of
``libsala.so``; there is no CPU or PyTorch fallback: if the library is missing
the first call raises.  Outputs and scratch buffers not passed by the caller are
allocated with torch (device memory is plumbing here).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "SalaError", "load_library", "lightning_prefill", "lightning_prefill_workspace",
    "lightning_prefill_noalloc", "lightning_projection", "lightning_prefill_prepared",
    "lightning_decode", "sparse_select", "sparse_select_workspace", "sparse_select_head_softmax_workspace", "sparse_attn",
    "sparse_attn_workspace",
    "get_device_error", "debug_bounds_line", "selftest_wait_timeout", "sparse_decode", "sparse_decode_workspace",
    "sparse_block_means", "lightning_state", "state_prefix_sum", "status_string", "version",
    "set_tracing",
    "LIB_PATH",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsala.so")
# SALA_LIBRARY=debug loads libsala_debug.so (the same kernels with device index checks,
# built with SALA_DEBUG); any other non-empty value is a path to the library
LIB_DEBUG_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsala_debug.so")
SALA_F32, SALA_BF16 = 0, 1
_lib = None


class SalaError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn} failed: {text} ({status})")
        self.status = status


_TRACE = os.environ.get("SALA_NVTX", "") not in ("", "0")


def set_tracing(on: bool = True) -> None:
    """Wrap every compute call of the library in an NVTX range named after its C entry
    point, for profiler timelines (SALA_NVTX=1 at import does the same).  Off by
    default: the calls are then made directly."""
    global _TRACE
    _TRACE = bool(on)


class _Lib:
    """The loaded libsala: attribute access goes to the C library; with tracing on, the
    compute entry points come back wrapped in NVTX ranges (workspace queries and the
    status helpers never are)."""

    _PLAIN = ("sala_status_string", "sala_version")

    def __init__(self, cdll):
        self._cdll = cdll

    def __getattr__(self, name):
        fn = getattr(self._cdll, name)
        if (not _TRACE or not name.startswith("sala_") or name.endswith("_workspace")
                or name in self._PLAIN):
            return fn

        def traced(*args):
            with torch.cuda.nvtx.range(name):
                return fn(*args)

        return traced


class SalaStrides(ctypes.Structure):
    _fields_ = [("b", ctypes.c_int64), ("t", ctypes.c_int64), ("h", ctypes.c_int64)]


def load_library(path: Optional[str] = None):
    """Load libsala.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    env = os.environ.get("SALA_LIBRARY", "")
    p = path or (LIB_DEBUG_PATH if env == "debug" else env) or LIB_PATH
    if not os.path.exists(p):
        raise OSError(f"libsala.so not found at {p}; build it with "
                      "`python -m sparse_attention_long_lightning_b200.build`")
    lib = ctypes.CDLL(p)
    vp, i, i64, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    S = SalaStrides
    lib.sala_status_string.argtypes = [i]
    lib.sala_status_string.restype = ctypes.c_char_p
    lib.sala_version.argtypes = []
    lib.sala_version.restype = ctypes.c_char_p
    lib.sala_lightning_prefill_workspace.argtypes = [i, i, i, i, i, i]
    lib.sala_lightning_prefill_workspace.restype = sz
    lib.sala_lightning_prefill.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, S, S, S, S,
                                           S, i, i64, f, f, i, vp, sz, i, vp]
    lib.sala_lightning_prefill.restype = i
    lib.sala_lightning_prefill_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, S,
                                                   S, S, S, S, i, i64, f, f, i, i, vp]
    lib.sala_lightning_prefill_noalloc.restype = i
    lib.sala_lightning_projection.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i64,
                                              S, S, S, S, i64, f, f, i, vp]
    lib.sala_lightning_projection.restype = i
    lib.sala_lightning_prefill_prepared.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, S, S, S, S,
                                                    S, i, i, vp, sz, vp]
    lib.sala_lightning_prefill_prepared.restype = i
    lib.sala_lightning_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, S, S, S, S,
                                          S, f, f, i, vp]
    lib.sala_lightning_decode.restype = i
    lib.sala_lightning_state.argtypes = [vp, vp, vp, vp, i, i, i, i, S, S, i, i64, f, f, i, vp, sz,
                                         i, vp]
    lib.sala_lightning_state.restype = i
    lib.sala_state_prefix_sum.argtypes = [vp, sz, i, sz, vp, i, vp]
    lib.sala_state_prefix_sum.restype = i
    lib.sala_sparse_select_workspace.argtypes = [i, i, i, i, i, i, i]
    lib.sala_sparse_select_workspace.restype = sz
    lib.sala_sparse_select.argtypes = [vp, vp, i, i, i, i, i, S, S, i, i, i, i, vp, vp, sz, i, vp]
    lib.sala_sparse_select.restype = i
    lib.sala_sparse_select_head_softmax_workspace.argtypes = [i, i, i, i, i, i]
    lib.sala_sparse_select_head_softmax_workspace.restype = sz
    lib.sala_sparse_select_head_softmax.argtypes = [vp, vp, i, i, i, i, i, S, S, i, i, i, i, vp,
                                                    vp, sz, i, vp]
    lib.sala_sparse_select_head_softmax.restype = i
    lib.sala_sparse_decode_workspace.argtypes = [i, i, i, i, i, i]
    lib.sala_sparse_decode_workspace.restype = sz
    lib.sala_sparse_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, S, S, S, S, S,
                                       i, i, i, i, f, vp, sz, i, vp]
    lib.sala_sparse_decode.restype = i
    lib.sala_sparse_block_means.argtypes = [vp, i, i, i, i, S, vp, i, i, vp]
    lib.sala_sparse_block_means.restype = i
    lib.sala_sparse_attn_workspace.argtypes = [i, i, i, i]
    lib.sala_sparse_attn_workspace.restype = sz
    lib.sala_sparse_attn.argtypes = [vp, vp, vp, vp, vp, i, vp, i, i, i, i, i, S, S, S, S, S, i, f,
                                     vp, sz, i, vp]
    lib.sala_sparse_attn.restype = i
    lib.sala_sparse_select_rows_workspace.argtypes = [i, i, i, i, i, i, i, i, i]
    lib.sala_sparse_select_rows_workspace.restype = sz
    lib.sala_sparse_select_rows.argtypes = [vp, vp, i, i, i, i, i, i, i, S, S, i, i, i, i, i, vp,
                                            vp, sz, i, vp]
    lib.sala_sparse_select_rows.restype = i
    lib.sala_sparse_attn_rows.argtypes = [vp, vp, vp, vp, vp, i, vp, i, i, i, i, i, i, i, S, S, S,
                                          S, S, i, f, vp, sz, i, vp]
    lib.sala_sparse_attn_rows.restype = i
    lib.sala_get_device_error.argtypes = [vp]
    lib.sala_get_device_error.restype = i
    lib.sala_debug_bounds_line.argtypes = []
    lib.sala_debug_bounds_line.restype = i
    lib.sala_selftest_wait_timeout.argtypes = [ctypes.c_longlong, vp]
    lib.sala_selftest_wait_timeout.restype = i
    _lib = _Lib(lib)
    return _lib


def status_string(status: int) -> str:
    return load_library().sala_status_string(int(status)).decode()


def version() -> str:
    return load_library().sala_version().decode()


def _check(fn: str, status: int):
    if status != 0:
        raise SalaError(fn, status, status_string(status))


def _p(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SALA_BF16
    if t.dtype == torch.float32:
        return SALA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _s4(t: Optional[torch.Tensor]) -> SalaStrides:
    """Element strides {b, t, h} of a [B, T, H, D] tensor (D stride must be 1)."""
    if t is None:
        return SalaStrides(0, 0, 0)
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError("expected a [B, T, H, D] tensor with unit stride along D")
    return SalaStrides(t.stride(0), t.stride(1), t.stride(2))


def _s3(t: Optional[torch.Tensor]) -> SalaStrides:
    """Element strides {b, -, h} of a [B, H, D] tensor."""
    if t is None:
        return SalaStrides(0, 0, 0)
    if t.dim() != 3 or t.stride(2) != 1:
        raise ValueError("expected a [B, H, D] tensor with unit stride along D")
    return SalaStrides(t.stride(0), 0, t.stride(1))


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")


def lightning_prefill_workspace(B, T, H, D, chunk=128, dtype=torch.bfloat16) -> int:
    dt = SALA_BF16 if dtype == torch.bfloat16 else SALA_F32
    return int(load_library().sala_lightning_prefill_workspace(B, T, H, D, chunk, dt))


def lightning_prefill(q, k, v, g=None, state=None, q_norm_w=None, k_norm_w=None, *, chunk=128,
                      pos0=0, rope_base=10000.0, eps=1e-6, out=None, workspace=None,
                      stream=None):
    """Lightning attention prefill.  q,k,v,g: [B,T,H,D].  `state` ([B,H,D,D] fp32) is the
    initial state, updated in place to the final state; None starts from zero.
    Returns (out [B,T,H,D], state)."""
    lib = load_library()
    _cuda(q, k, v, g, state, out)
    B, T, H, D = q.shape
    init_zero = 1 if state is None else 0
    if state is None:
        state = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
    if out is None:
        out = torch.empty((B, T, H, D), dtype=q.dtype, device=q.device)
    need = lightning_prefill_workspace(B, T, H, D, chunk, q.dtype)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib.sala_lightning_prefill(
        _p(q), _p(k), _p(v), _p(g), _p(out), _p(state), _p(q_norm_w), _p(k_norm_w), B, T, H, D,
        _s4(q), _s4(k), _s4(v), _s4(g), _s4(out), int(chunk), int(pos0), float(rope_base),
        float(eps), init_zero, _p(workspace), wsb, _dt(q), _stream(stream))
    _check("sala_lightning_prefill", st)
    return out, state


def lightning_prefill_noalloc(q, k, v, g, state, out, q_norm_w=None, k_norm_w=None, *, chunk=128,
                              pos0=0, rope_base=10000.0, eps=1e-6, init_zero=False, stream=None):
    """Lightning prefill through the entry point that allocates nothing.

    For callers that cannot give the library a workspace (a host framework that
    owns all device memory, or a serving loop whose pool is frozen): the library
    keeps the per-segment scratch in a fixed 16 MiB device array instead.  The
    caller passes preallocated `state` ([B,H,D,D] fp32, in/out) and `out`; with
    init_zero the incoming state is ignored.  Calls that may overlap on the GPU
    share that array and must be serialised.  B*H above 256 raises SalaError
    (SALA_ERR_WORKSPACE) for the bf16 / head_dim 128 / chunk 128 path."""
    lib = load_library()
    _cuda(q, k, v, g, state, out)
    B, T, H, D = q.shape
    st = lib.sala_lightning_prefill_noalloc(
        _p(q), _p(k), _p(v), _p(g), _p(out), _p(state), _p(q_norm_w), _p(k_norm_w), B, T, H, D,
        _s4(q), _s4(k), _s4(v), _s4(g), _s4(out), int(chunk), int(pos0), float(rope_base),
        float(eps), 1 if init_zero else 0, _dt(q), _stream(stream))
    _check("sala_lightning_prefill_noalloc", st)
    return out, state


def lightning_projection(x, w, q_norm_w=None, k_norm_w=None, *, heads, head_dim=128, pos0=0,
                         rope_base=10000.0, eps=1e-6, out=None, stream=None):
    """Input projection of a Lightning layer with its preparation fused in.

    x: [B, T, hidden] bf16 (rows packed: x.stride(0) == T * x.stride(1)); w: [4 H D,
    hidden] bf16 contiguous (q heads, then k, v, g).  Returns (qh, kh, v, gate), each
    [B, T, H, D]: qh, kh fp16 (RMSNorm, norm weight, RoPE at pos0 + t), v bf16, gate =
    sigmoid(g) fp16.  `out` may give the four output tensors."""
    lib = load_library()
    _cuda(x, w, q_norm_w, k_norm_w)
    B, T, hidden = x.shape
    H, D = int(heads), int(head_dim)
    if x.dtype != torch.bfloat16 or w.dtype != torch.bfloat16:
        raise TypeError("x and w must be bf16")
    if w.shape != (4 * H * D, hidden) or not w.is_contiguous():
        raise ValueError("w must be a contiguous [4 H D, hidden] tensor")
    if x.stride(2) != 1 or (B > 1 and x.stride(0) != T * x.stride(1)):
        raise ValueError("x rows must be packed with unit stride along hidden")
    if out is None:
        shape = (B, T, H, D)
        out = (torch.empty(shape, dtype=torch.float16, device=x.device),
               torch.empty(shape, dtype=torch.float16, device=x.device),
               torch.empty(shape, dtype=torch.bfloat16, device=x.device),
               torch.empty(shape, dtype=torch.float16, device=x.device))
    qh, kh, v, gate = out
    _cuda(qh, kh, v, gate)
    st = lib.sala_lightning_projection(
        _p(x), _p(w), _p(q_norm_w), _p(k_norm_w), _p(qh), _p(kh), _p(v), _p(gate), B, T, hidden,
        H, D, x.stride(1), _s4(qh), _s4(kh), _s4(v), _s4(gate), int(pos0), float(rope_base),
        float(eps), SALA_BF16, _stream(stream))
    _check("sala_lightning_projection", st)
    return qh, kh, v, gate


def lightning_prefill_prepared(qh, kh, v, gate=None, state=None, *, chunk=128, out=None,
                               workspace=None, stream=None):
    """Lightning prefill on prepared operands (lightning_projection's outputs): qh, kh
    [B,T,H,D] fp16 already normalised and rotated, v bf16, gate fp16 multiplier (or
    None).  `state` as in lightning_prefill.  Returns (out [B,T,H,D] bf16, state)."""
    lib = load_library()
    _cuda(qh, kh, v, gate, state, out)
    B, T, H, D = qh.shape
    if qh.dtype != torch.float16 or kh.dtype != torch.float16 or v.dtype != torch.bfloat16:
        raise TypeError("qh, kh must be fp16 and v bf16")
    if gate is not None and gate.dtype != torch.float16:
        raise TypeError("gate must be fp16 (the sigmoid multiplier)")
    init_zero = 1 if state is None else 0
    if state is None:
        state = torch.empty((B, H, D, D), dtype=torch.float32, device=qh.device)
    if out is None:
        out = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=qh.device)
    need = lightning_prefill_workspace(B, T, H, D, chunk, torch.bfloat16)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=qh.device)
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib.sala_lightning_prefill_prepared(
        _p(qh), _p(kh), _p(v), _p(gate), _p(out), _p(state), B, T, H, D, _s4(qh), _s4(kh),
        _s4(v), _s4(gate), _s4(out), int(chunk), init_zero, _p(workspace), wsb, _stream(stream))
    _check("sala_lightning_prefill_prepared", st)
    return out, state


def lightning_decode(q, k, v, g, state, pos, q_norm_w=None, k_norm_w=None, *, rope_base=10000.0,
                     eps=1e-6, out=None, stream=None):
    """One decode step.  q,k,v,g: [B,H,D]; state [B,H,D,D] fp32 (updated in place);
    pos: [B] int32 CUDA tensor.  Returns out [B,H,D]."""
    lib = load_library()
    _cuda(q, k, v, g, state, pos, out)
    B, H, D = q.shape
    if pos.dtype != torch.int32:
        raise TypeError("pos must be int32")
    if out is None:
        out = torch.empty((B, H, D), dtype=q.dtype, device=q.device)
    st = lib.sala_lightning_decode(
        _p(q), _p(k), _p(v), _p(g), _p(out), _p(state), _p(q_norm_w), _p(k_norm_w), _p(pos), B, H,
        D, _s3(q), _s3(k), _s3(v), _s3(g), _s3(out), float(rope_base), float(eps), _dt(q),
        _stream(stream))
    _check("sala_lightning_decode", st)
    return out


def lightning_state(k, v, state=None, k_norm_w=None, *, chunk=128, pos0=0, rope_base=10000.0,
                    eps=1e-6, workspace=None, stream=None):
    """Segment state sum_t kh_t v_t^T of k, v [B,T,H,D] (added to `state` [B,H,D,D] fp32
    when given, else from zero).  Returns the state."""
    lib = load_library()
    _cuda(k, v, state, k_norm_w, workspace)
    B, T, H, D = k.shape
    init_zero = state is None
    if state is None:
        state = torch.empty((B, H, D, D), dtype=torch.float32, device=k.device)
    need = lightning_prefill_workspace(B, T, H, D, chunk) if k.dtype == torch.bfloat16 else 0
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=k.device)
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib.sala_lightning_state(_p(k), _p(v), _p(state), _p(k_norm_w), B, T, H, D, _s4(k),
                                  _s4(v), int(chunk), int(pos0), float(rope_base), float(eps),
                                  int(init_zero), _p(workspace), wsb, _dt(k), _stream(stream))
    _check("sala_lightning_state", st)
    return state


def state_prefix_sum(gathered, count, out, accumulate=True, stream=None):
    """out (+)= sum of gathered[0..count-1] (fp32 tensors of out's size)."""
    lib = load_library()
    _cuda(gathered, out)
    n = out.numel()
    if gathered.dtype != torch.float32 or out.dtype != torch.float32:
        raise TypeError("float32 states expected")
    if not gathered.is_contiguous() or not out.is_contiguous() or gathered[0].numel() != n:
        raise ValueError("gathered must be [count, *out.shape] contiguous")
    st = lib.sala_state_prefix_sum(_p(gathered), n, int(count), n, _p(out), int(accumulate),
                                   _stream(stream))
    _check("sala_state_prefix_sum", st)
    return out


def sparse_select_workspace(B, T, Hq, Hkv, D, block=64, topk=64) -> int:
    return int(load_library().sala_sparse_select_workspace(B, T, Hq, Hkv, D, block, topk))


def sparse_select_head_softmax_workspace(B, T, Hq, Hkv, D, block=64) -> int:
    return int(load_library().sala_sparse_select_head_softmax_workspace(B, T, Hq, Hkv, D, block))


def sparse_select_rows_workspace(B, Tq, Tk, Hq, Hkv, D, block=64, topk=64,
                                 score="group_sum") -> int:
    mode = 1 if score == "head_softmax" else 0
    return int(load_library().sala_sparse_select_rows_workspace(B, Tq, Tk, Hq, Hkv, D, block,
                                                                topk, mode))


def _q_window(q, k, q_pos0):
    """(Tq, qpos0, Tk) of a call whose q rows may be a window of k's positions; None when
    q covers all of k's positions from 0 (the whole-sequence entry points)."""
    Tq, Tk = q.shape[1], k.shape[1]
    if q_pos0 is None:
        if Tq != Tk:
            raise ValueError("q and k differ in length: pass q_pos0, the position of q's row 0")
        return None
    if not 0 <= int(q_pos0) <= Tk - Tq:
        raise ValueError("the q rows must lie inside k's positions")
    return Tq, int(q_pos0), Tk


def sparse_select(q, k, *, topk=64, n_init=1, n_local=2, block=64, out=None, workspace=None,
                  stream=None, score="group_sum", q_pos0=None):
    """Block selection.  q [B,T,Hq,D], k [B,T,Hkv,D] -> idx [B,Hkv,T,n_init+topk+n_local] int32.
    score="group_sum" (sala_sparse_select) or "head_softmax" (sala_sparse_select_head_softmax).
    With q_pos0, q holds Tq rows at positions q_pos0 .. q_pos0 + Tq - 1 of a sequence whose
    keys k [B,Tk,Hkv,D] cover 0 .. Tk - 1 (sala_sparse_select_rows); idx is [B,Hkv,Tq,n_sel]."""
    if score not in ("group_sum", "head_softmax"):
        raise ValueError("score must be 'group_sum' or 'head_softmax'")
    lib = load_library()
    _cuda(q, k, out, workspace)
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    n_sel = n_init + topk + n_local
    if out is None:
        out = torch.empty((B, Hkv, T, n_sel), dtype=torch.int32, device=q.device)
    hsm = score == "head_softmax"
    win = _q_window(q, k, q_pos0)
    if win is not None:
        Tq, qp, Tk = win
        need = sparse_select_rows_workspace(B, Tq, Tk, Hq, Hkv, D, block, topk, score)
        if workspace is None and need:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
        st = lib.sala_sparse_select_rows(_p(q), _p(k), B, Tq, qp, Tk, Hq, Hkv, D, _s4(q), _s4(k),
                                         int(block), int(topk), int(n_init), int(n_local),
                                         1 if hsm else 0, _p(out), _p(workspace), wsb, _dt(q),
                                         _stream(stream))
        _check("sala_sparse_select_rows", st)
        return out
    need = (sparse_select_head_softmax_workspace(B, T, Hq, Hkv, D, block) if hsm
            else sparse_select_workspace(B, T, Hq, Hkv, D, block, topk))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    fn = lib.sala_sparse_select_head_softmax if hsm else lib.sala_sparse_select
    st = fn(_p(q), _p(k), B, T, Hq, Hkv, D, _s4(q), _s4(k), int(block), int(topk), int(n_init),
            int(n_local), _p(out), _p(workspace), wsb, _dt(q), _stream(stream))
    _check("sala_sparse_select_head_softmax" if hsm else "sala_sparse_select", st)
    return out


def sparse_attn_workspace(B, T, Hkv, D) -> int:
    return int(load_library().sala_sparse_attn_workspace(B, T, Hkv, D))


def sparse_attn(q, k, v, idx, g=None, *, block=64, scale=0.0, out=None, workspace=None,
                stream=None, q_pos0=None):
    """Block-sparse attention.  q,g [B,T,Hq,D]; k,v [B,T,Hkv,D]; idx [B,Hkv,T,n_sel] int32.
    With q_pos0, q, g, idx and the output hold Tq rows at positions q_pos0 .. q_pos0 + Tq - 1
    of a sequence whose k, v [B,Tk,Hkv,D] cover 0 .. Tk - 1 (sala_sparse_attn_rows)."""
    lib = load_library()
    _cuda(q, k, v, idx, g, out, workspace)
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    if idx.dtype != torch.int32 or not idx.is_contiguous():
        raise ValueError("idx must be a contiguous int32 tensor")
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    win = _q_window(q, k, q_pos0)
    if win is not None:
        Tq, qp, Tk = win
        need = sparse_attn_workspace(B, Tk, Hkv, D)
        if workspace is None and need:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
        st = lib.sala_sparse_attn_rows(_p(q), _p(k), _p(v), _p(g), _p(idx), int(idx.shape[-1]),
                                       _p(out), B, Tq, qp, Tk, Hq, Hkv, D, _s4(q), _s4(k), _s4(v),
                                       _s4(g), _s4(out), int(block), float(scale), _p(workspace),
                                       wsb, _dt(q), _stream(stream))
        _check("sala_sparse_attn_rows", st)
        return out
    need = sparse_attn_workspace(B, T, Hkv, D)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib.sala_sparse_attn(_p(q), _p(k), _p(v), _p(g), _p(idx), int(idx.shape[-1]), _p(out), B,
                              T, Hq, Hkv, D, _s4(q), _s4(k), _s4(v), _s4(g), _s4(out), int(block),
                              float(scale), _p(workspace), wsb, _dt(q), _stream(stream))
    _check("sala_sparse_attn", st)
    return out


def sparse_decode_workspace(B, Tmax, Hq, Hkv, D, n_sel) -> int:
    return int(load_library().sala_sparse_decode_workspace(B, Tmax, Hq, Hkv, D, n_sel))


def sparse_decode(q, k_cache, v_cache, kbar, pos, g=None, *, topk=64, n_init=1, n_local=2,
                  block=64, scale=0.0, out=None, idx_out=None, workspace=None, stream=None):
    """One sparse-layer decode step.  q,g [B,Hq,D]; k_cache,v_cache [B,Tmax,Hkv,D] with the
    new token already at row pos[b]; kbar [B,Tmax/64,Hkv,D] fp32 block-mean cache (updated
    when the token completes a block); pos [B] int32 CUDA.  Returns out [B,Hq,D]."""
    lib = load_library()
    _cuda(q, k_cache, v_cache, kbar, pos, g, out, idx_out, workspace)
    B, Hq, D = q.shape
    Tmax, Hkv = k_cache.shape[1], k_cache.shape[2]
    if pos.dtype != torch.int32:
        raise TypeError("pos must be int32")
    if kbar.dtype != torch.float32 or not kbar.is_contiguous():
        raise ValueError("kbar must be a contiguous float32 tensor")
    n_sel = n_init + topk + n_local
    if out is None:
        out = torch.empty((B, Hq, D), dtype=q.dtype, device=q.device)
    if idx_out is not None and (idx_out.dtype != torch.int32 or not idx_out.is_contiguous()):
        raise ValueError("idx_out must be a contiguous int32 tensor")
    need = sparse_decode_workspace(B, Tmax, Hq, Hkv, D, n_sel)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib.sala_sparse_decode(
        _p(q), _p(k_cache), _p(v_cache), _p(g), _p(kbar), _p(pos), _p(out), _p(idx_out), B, Tmax,
        Hq, Hkv, D, _s3(q), _s4(k_cache), _s4(v_cache), _s3(g), _s3(out), int(block), int(topk),
        int(n_init), int(n_local), float(scale), _p(workspace), wsb, _dt(q), _stream(stream))
    _check("sala_sparse_decode", st)
    return out


def sparse_block_means(k, kbar=None, *, kbar_blocks=None, stream=None):
    """Block means of the complete blocks of k [B,T,Hkv,D] into kbar [B,kbar_blocks,Hkv,D]
    fp32 (allocated with kbar_blocks = T // 64 when not given)."""
    lib = load_library()
    _cuda(k, kbar)
    B, T, Hkv, D = k.shape
    if kbar is None:
        nb = T // 64 if kbar_blocks is None else int(kbar_blocks)
        kbar = torch.zeros((B, nb, Hkv, D), dtype=torch.float32, device=k.device)
    if kbar.dtype != torch.float32 or not kbar.is_contiguous():
        raise ValueError("kbar must be a contiguous float32 tensor")
    st = lib.sala_sparse_block_means(_p(k), B, T, Hkv, D, _s4(k), _p(kbar), int(kbar.shape[1]),
                                     _dt(k), _stream(stream))
    _check("sala_sparse_block_means", st)
    return kbar


def selftest_wait_timeout(cycles=20_000_000, stream=None):
    """Run the bounded-wait failure path on the GPU: a wait that can never complete
    gives up after `cycles` clock cycles and sets SALA_ERR_TIMEOUT (read it with
    get_device_error)."""
    _check("sala_selftest_wait_timeout",
           load_library().sala_selftest_wait_timeout(int(cycles), _stream(stream)))


def get_device_error(stream=None) -> int:
    """Synchronise the stream and read/clear the device error word (0 = none)."""
    return int(load_library().sala_get_device_error(_stream(stream)))


def debug_bounds_line() -> int:
    """Source line of the first failed device index check since the last call (0: none;
    -1: the release library, which has no checks).  Clears it."""
    return int(load_library().sala_debug_bounds_line())
