"""GPU: guard bands around every buffer a libsala call writes.

Each output, in/out state and workspace is a view into a larger buffer whose head and
tail are filled with a sentinel bit pattern; after the call the sentinels must be
intact, so a write outside the buffer the caller handed over is caught (the checks the
library cannot make about its own kernels' index arithmetic).  Ragged and small shapes.
"""
import pytest
import torch

from sparse_attention_long_lightning_b200 import inputs

pytestmark = pytest.mark.gpu

sala = pytest.importorskip("sparse_attention_long_lightning_b200")
DEV = "cuda"
GUARD_BYTES = 64 * 1024
PATTERN = 0x5A  # sentinel byte


class Guarded:
    """A tensor view with GUARD_BYTES of sentinel on both sides (16-byte aligned)."""

    def __init__(self, shape, dtype, init=None):
        esz = torch.empty((), dtype=dtype).element_size()
        n = 1
        for s in shape:
            n *= s
        self.nbytes = n * esz
        self.raw = torch.full((GUARD_BYTES + self.nbytes + GUARD_BYTES,), PATTERN,
                              dtype=torch.uint8, device=DEV)
        self.view = self.raw[GUARD_BYTES:GUARD_BYTES + self.nbytes].view(dtype).view(shape)
        if init is not None:
            self.view.copy_(init)

    def intact(self):
        head = self.raw[:GUARD_BYTES]
        tail = self.raw[GUARD_BYTES + self.nbytes:]
        return bool((head == PATTERN).all()) and bool((tail == PATTERN).all())


def _ws(nbytes):
    return Guarded((max(int(nbytes), 1),), torch.uint8)


@pytest.mark.parametrize("T,H,D,chunk", [(777, 4, 128, 128), (333, 3, 64, 64), (130, 2, 128, 64)])
def test_lightning_prefill_writes_stay_inside(T, H, D, chunk):
    x = inputs.lightning_inputs(1, T, H, D, seed=T + H, device=DEV)
    out = Guarded((1, T, H, D), torch.bfloat16)
    state = Guarded((1, H, D, D), torch.float32, init=torch.zeros((1, H, D, D)))
    ws = _ws(sala.lightning_prefill_workspace(1, T, H, D, chunk))
    sala.lightning_prefill(x.q, x.k, x.v, x.g, state.view, chunk=chunk, out=out.view,
                           workspace=ws.view)
    torch.cuda.synchronize()
    assert sala.get_device_error() == 0
    assert out.intact() and state.intact() and ws.intact()


def test_lightning_decode_writes_stay_inside():
    B, H, D = 5, 4, 128
    S0 = inputs.decode_state(B, H, D, seed=5, device=DEV)
    q, k, v, g = inputs.decode_tokens(B, H, D, seed=5, step=0, device=DEV)
    state = Guarded((B, H, D, D), torch.float32, init=S0)
    out = Guarded((B, H, D), torch.bfloat16)
    pos = torch.arange(B, dtype=torch.int32, device=DEV) * 97
    sala.lightning_decode(q, k, v, g, state.view, pos, out=out.view)
    torch.cuda.synchronize()
    assert sala.get_device_error() == 0
    assert out.intact() and state.intact()


@pytest.mark.parametrize("topk,score", [(8, "group_sum"), (100, "group_sum"),
                                        (8, "head_softmax")])
def test_select_and_attn_writes_stay_inside(topk, score):
    T, Hq, Hkv, D = 64 * 30 + 13, 16, 2, 128
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=topk + 7, device=DEV, gate=True)
    n_sel = 1 + topk + 2
    idx = Guarded((1, Hkv, T, n_sel), torch.int32)
    need = (sala.sparse_select_head_softmax_workspace(1, T, Hq, Hkv, D) if score == "head_softmax"
            else sala.sparse_select_workspace(1, T, Hq, Hkv, D, 64, topk))
    ws = _ws(need)
    sala.sparse_select(s.q, s.k, topk=topk, out=idx.view, workspace=ws.view, score=score)
    out = Guarded((1, T, Hq, D), torch.bfloat16)
    wsa = _ws(sala.sparse_attn_workspace(1, T, Hkv, D))
    sala.sparse_attn(s.q, s.k, s.v, idx.view, s.g, out=out.view, workspace=wsa.view)
    torch.cuda.synchronize()
    assert sala.get_device_error() == 0
    assert idx.intact() and ws.intact() and out.intact() and wsa.intact()


def test_sparse_decode_and_block_means_writes_stay_inside():
    B, Tmax, Hq, Hkv, D = 3, 64 * 12, 16, 2, 128
    gen = inputs.generator(31, DEV)
    kc = inputs.randn((B, Tmax, Hkv, D), gen, device=DEV)
    vc = inputs.randn((B, Tmax, Hkv, D), gen, device=DEV)
    q = inputs.randn((B, Hq, D), gen, device=DEV)
    g = inputs.randn((B, Hq, D), gen, device=DEV)
    kbar = Guarded((B, Tmax // 64, Hkv, D), torch.float32,
                   init=torch.zeros((B, Tmax // 64, Hkv, D)))
    sala.sparse_block_means(kc[:, :64 * 7 + 5], kbar.view)
    pos = torch.tensor([64 * 7 + 63, 64 * 11 + 2, 17], dtype=torch.int32, device=DEV)
    out = Guarded((B, Hq, D), torch.bfloat16)
    idx = Guarded((B, Hkv, 67), torch.int32)
    ws = _ws(sala.sparse_decode_workspace(B, Tmax, Hq, Hkv, D, 67))
    sala.sparse_decode(q, kc, vc, kbar.view, pos, g, out=out.view, idx_out=idx.view,
                       workspace=ws.view)
    torch.cuda.synchronize()
    assert sala.get_device_error() == 0
    assert kbar.intact() and out.intact() and idx.intact() and ws.intact()


@pytest.mark.parametrize("score", ["group_sum", "head_softmax"])
def test_row_window_calls_write_stay_inside(score):
    """Selection and attention over a window of query rows (row-window entry points)."""
    T, Hq, Hkv, D, topk = 64 * 40 + 29, 16, 2, 128, 16
    a, b = 64 * 11 + 5, 64 * 31 + 3
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=61, device=DEV, gate=True)
    n_sel = 1 + topk + 2
    idx = Guarded((1, Hkv, b - a, n_sel), torch.int32)
    ws = _ws(sala.sparse_select_rows_workspace(1, b - a, T, Hq, Hkv, D, 64, topk, score))
    sala.sparse_select(s.q[:, a:b], s.k, topk=topk, out=idx.view, workspace=ws.view,
                       score=score, q_pos0=a)
    out = Guarded((1, b - a, Hq, D), torch.bfloat16)
    wsa = _ws(sala.sparse_attn_workspace(1, T, Hkv, D))
    sala.sparse_attn(s.q[:, a:b], s.k, s.v, idx.view, s.g[:, a:b], out=out.view,
                     workspace=wsa.view, q_pos0=a)
    torch.cuda.synchronize()
    assert sala.get_device_error() == 0
    assert idx.intact() and ws.intact() and out.intact() and wsa.intact()


def test_projection_and_prepared_prefill_writes_stay_inside():
    """The fused projection's four outputs, then the prepared prefill's output, state and
    workspace, on ragged rows (2 x 301 tokens: a partial last tile)."""
    B, T, hidden, H, D = 2, 301, 256, 2, 128
    gen = inputs.generator(62, DEV)
    x = inputs.randn((B, T, hidden), gen, device=DEV)
    w = inputs.randn((4 * H * D, hidden), gen, device=DEV, scale=hidden ** -0.5)
    outs = (Guarded((B, T, H, D), torch.float16), Guarded((B, T, H, D), torch.float16),
            Guarded((B, T, H, D), torch.bfloat16), Guarded((B, T, H, D), torch.float16))
    qh, kh, v, gate = sala.lightning_projection(x, w, heads=H, head_dim=D, pos0=5,
                                                out=tuple(o.view for o in outs))
    state = Guarded((B, H, D, D), torch.float32, init=torch.zeros((B, H, D, D)))
    y = Guarded((B, T, H, D), torch.bfloat16)
    ws = _ws(sala.lightning_prefill_workspace(B, T, H, D, 128))
    sala.lightning_prefill_prepared(qh, kh, v, gate, state.view, out=y.view, workspace=ws.view)
    torch.cuda.synchronize()
    assert sala.get_device_error() == 0
    assert all(o.intact() for o in outs) and state.intact() and y.intact() and ws.intact()


def test_state_only_and_noalloc_writes_stay_inside():
    """The state-only pass (sequence-parallel Lightning) and the allocation-free prefill."""
    T, H, D = 128 * 3 + 77, 4, 128
    x = inputs.lightning_inputs(1, T, H, D, seed=63, device=DEV)
    state = Guarded((1, H, D, D), torch.float32, init=torch.zeros((1, H, D, D)))
    ws = _ws(sala.lightning_prefill_workspace(1, T, H, D, 128))
    sala.lightning_state(x.k, x.v, state.view, workspace=ws.view, pos0=128)
    st2 = Guarded((1, H, D, D), torch.float32, init=torch.zeros((1, H, D, D)))
    out = Guarded((1, T, H, D), torch.bfloat16)
    sala.lightning_prefill_noalloc(x.q, x.k, x.v, x.g, st2.view, out.view)
    torch.cuda.synchronize()
    assert sala.get_device_error() == 0
    assert state.intact() and ws.intact() and st2.intact() and out.intact()
