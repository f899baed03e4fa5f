"""GPU parity: the Lightning layer's input projection with the fused QK-norm / RoPE / gate
epilogue (sala_lightning_projection) and the Lightning prefill on its prepared operands
(sala_lightning_prefill_prepared), against the fp64 oracle.

Weights are seeded synthetic N(0, 1/hidden) values (the pages publish none).  The
projection multiplies bf16 x and W with fp32 accumulation; qh, kh are stored as fp16
(rounding 2^-12 relative), as is the gate multiplier sigmoid(g) (a value in (0, 1)); v as
bf16 (half an ulp allowed, as everywhere).
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_long_lightning_b200 import inputs
from tests._parity import TOL_BF16, raw_rel_err, rel_err

pytestmark = pytest.mark.gpu

sala = pytest.importorskip("sparse_attention_long_lightning_b200")
DEV = "cuda"


def _np(t):
    return t.detach().double().cpu().numpy()


def _layer(B, T, hidden, H, D, seed, weights=True):
    gen = inputs.generator(seed)
    x = inputs.randn((B, T, hidden), gen)
    w = inputs.randn((4 * H * D, hidden), gen, scale=hidden ** -0.5)
    qw = kw = None
    if weights:
        qw = 1.0 + 0.1 * inputs.randn((D,), gen, torch.float32)
        kw = 1.0 + 0.1 * inputs.randn((D,), gen, torch.float32)
    return x, w, qw, kw


def _check_projection(outs, ref):
    qh, kh, v, gate = outs
    rq, rk, rv, rg = ref
    assert qh.dtype == torch.float16 and v.dtype == torch.bfloat16 and gate.dtype == torch.float16
    assert raw_rel_err(_np(qh), rq) <= TOL_BF16
    assert raw_rel_err(_np(kh), rk) <= TOL_BF16
    assert rel_err(_np(v), rv, True) <= TOL_BF16
    assert raw_rel_err(_np(gate), rg) <= TOL_BF16


@pytest.mark.parametrize("B,T,hidden,H,D,weights,pos0", [
    (2, 300, 512, 4, 128, True, 7),      # ragged rows (600 = 4 tiles + 88), 2 column tiles/section
    (1, 129, 256, 4, 64, False, 0),      # head_dim 64: four heads per 256-wide tile
    (3, 77, 192, 2, 128, True, 100000),  # a far position, three sequences in one tile
])
def test_projection_matches_oracle(B, T, hidden, H, D, weights, pos0):
    x, w, qw, kw = _layer(B, T, hidden, H, D, seed=4000 + T, weights=weights)
    outs = sala.lightning_projection(x.cuda(), w.cuda(), None if qw is None else qw.cuda(),
                                     None if kw is None else kw.cuda(), heads=H, head_dim=D,
                                     pos0=pos0)
    assert sala.get_device_error() == 0
    ref = oracle.lightning_projection(_np(x), _np(w), None if qw is None else _np(qw),
                                      None if kw is None else _np(kw), H=H, D=D, pos0=pos0)
    _check_projection(outs, ref)


def test_projection_full_width_sampled_rows():
    """hidden 4096, 32 heads of 128 (the 9B model's attention width), 4096 tokens: the
    whole projection on the GPU, 48 sampled rows (each at its own position) against the
    oracle."""
    B, T, hidden, H, D = 1, 4096, 4096, 32, 128
    x, w, qw, kw = _layer(B, T, hidden, H, D, seed=4100)
    xd = x.cuda()
    outs = sala.lightning_projection(xd, w.cuda(), qw.cuda(), kw.cuda(), heads=H, head_dim=D,
                                     pos0=11)
    assert sala.get_device_error() == 0
    rows = np.unique(np.concatenate([[0, 1, 127, 128, T - 1],
                                     np.random.default_rng(3).choice(T, 43, replace=False)]))
    wn, qn, kn = _np(w), _np(qw), _np(kw)
    for name, i in (("qh", 0), ("kh", 1), ("v", 2), ("gate", 3)):
        got = np.stack([_np(outs[i][:, r]) for r in rows], axis=1)
        want = np.concatenate([oracle.lightning_projection(_np(x[:, r:r + 1]), wn, qn, kn, H=H,
                                                           D=D, pos0=11 + int(r))[i]
                               for r in rows], axis=1)
        err = rel_err(got, want, True) if i == 2 else raw_rel_err(got, want)
        assert err <= TOL_BF16, (name, err)


@pytest.mark.parametrize("T", [1, 127, 128 * 9 + 45])
def test_prepared_prefill_matches_oracle(T):
    """The prepared prefill against the oracle's recurrence on the same (GPU-prepared)
    operands, with a start state."""
    B, hidden, H, D = 2, 256, 2, 128
    x, w, qw, kw = _layer(B, T, hidden, H, D, seed=4200 + T)
    qh, kh, v, gate = sala.lightning_projection(x.cuda(), w.cuda(), qw.cuda(), kw.cuda(),
                                                heads=H, head_dim=D, pos0=3)
    gen = inputs.generator(4201)
    S0 = inputs.randn((B, H, D, D), gen, torch.float32, scale=0.05)
    y, S = sala.lightning_prefill_prepared(qh, kh, v, gate, S0.cuda().clone())
    assert sala.get_device_error() == 0
    yr, Sr = oracle.lightning_recurrent_prepared(_np(qh), _np(kh), _np(v), _np(gate), _np(S0))
    assert rel_err(_np(y), yr, True) <= TOL_BF16
    assert rel_err(_np(S), Sr, False) <= TOL_BF16


def test_projection_then_prefill_end_to_end():
    """Hidden states -> projection -> prepared prefill, against the oracle's projection
    and recurrence in fp64.  Between the two calls v is an activation stored in bf16 (its
    rounding, 2^-9 relative, passes through the recurrence), so the reference pipeline
    stores the oracle's v in bf16 at the same point; qh, kh and the gate stay exact in the
    reference (the GPU keeps them in fp16)."""
    B, T, hidden, H, D = 1, 1500, 512, 4, 128
    x, w, qw, kw = _layer(B, T, hidden, H, D, seed=4300)
    qh, kh, v, gate = sala.lightning_projection(x.cuda(), w.cuda(), qw.cuda(), kw.cuda(),
                                                heads=H, head_dim=D, pos0=0)
    y, S = sala.lightning_prefill_prepared(qh, kh, v, gate)
    assert sala.get_device_error() == 0
    rq, rk, rv, rg = oracle.lightning_projection(_np(x), _np(w), _np(qw), _np(kw), H=H, D=D)
    rv = torch.from_numpy(rv).to(torch.bfloat16).double().numpy()  # the activation dtype
    yr, Sr = oracle.lightning_recurrent_prepared(rq, rk, rv, rg)
    assert rel_err(_np(y), yr, True) <= TOL_BF16
    assert rel_err(_np(S), Sr, False) <= TOL_BF16


def test_prepared_prefill_scaled_v_and_no_gate():
    """v far from unit scale (the per-segment power-of-two scale) and no gate."""
    B, T, hidden, H, D = 1, 128 * 6 + 3, 256, 2, 128
    x, w, qw, kw = _layer(B, T, hidden, H, D, seed=4400)
    qh, kh, v, _ = sala.lightning_projection(x.cuda(), w.cuda(), qw.cuda(), kw.cuda(), heads=H,
                                             head_dim=D)
    for scale in (1e-6, 1e4):
        vs = (v.float() * scale).to(torch.bfloat16)
        y, S = sala.lightning_prefill_prepared(qh, kh, vs, None)
        assert sala.get_device_error() == 0
        yr, Sr = oracle.lightning_recurrent_prepared(_np(qh), _np(kh), _np(vs))
        assert rel_err(_np(y), yr, True) <= TOL_BF16
        assert rel_err(_np(S), Sr, False) <= TOL_BF16


def test_projection_rejects_bad_shapes():
    x = torch.zeros((1, 8, 96), dtype=torch.bfloat16, device=DEV)    # hidden not a multiple of 64
    w = torch.zeros((4 * 2 * 128, 96), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(sala.SalaError) as e:
        sala.lightning_projection(x, w, heads=2)
    assert e.value.status == 2
    x = torch.zeros((1, 8, 128), dtype=torch.bfloat16, device=DEV)
    w = torch.zeros((4 * 1 * 128, 128), dtype=torch.bfloat16, device=DEV)   # H*D = 128
    with pytest.raises(sala.SalaError) as e:
        sala.lightning_projection(x, w, heads=1)
    assert e.value.status == 2
