"""GPU parity for bf16 inputs far from unit scale.

bf16 spans about 2^-133 .. 2^128, but the tensor-core Lightning passes and the block-sparse
attention multiply v in fp16, whose normal range is 2^-14 .. 65504.  The kernels scale v
by a power of two chosen from the largest |v| of each token segment (Lightning) or of each
(sequence, KV head) (sparse attention) and undo it in the fp32 epilogue; the sparse decode
keeps v in bf16 and splits P into two bf16 parts.  So v (and g) scaled by 1e-6, 1e-3 and
1e3, and a v holding one value of 1e5 or 1e6 among N(0,1) values, must meet the same bound
as unit-scale inputs (max|err| / rms(ref) <= 1e-2, against the fp64 oracle).  Only a
non-finite input raises SALA_ERR_RANGE.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_long_lightning_b200 import inputs
from tests._parity import TOL_BF16, TOL_F32, rel_err

pytestmark = pytest.mark.gpu

sala = pytest.importorskip("sparse_attention_long_lightning_b200")
DEV = "cuda"
SALA_ERR_RANGE = 6
CASES = [1e-6, 1e-3, 1e3, "spike1e5", "spike1e6"]


def _np(t):
    return t.detach().double().cpu().numpy()


def _rescale(x, case, where):
    """x times the case's scale, or x with one entry (index `where`) set to 1e5 / 1e6."""
    y = x.float().clone()
    if isinstance(case, str):
        y[where] = float(case[len("spike"):])
    else:
        y *= case
    return y.to(x.dtype)


@pytest.mark.parametrize("case", CASES)
def test_lightning_tensor_core_scaled_v(case):
    """bf16, head_dim 128, chunk 128 (state pass + scan + output pass): 14 segments of one
    chunk per head, so a spike leaves most segments unscaled and scales its own."""
    B, T, H, D = 1, 64 * 27 + 5, 2, 128
    x = inputs.lightning_inputs(B, T, H, D, seed=3100)
    v = _rescale(x.v, case, (0, 777, 1, 9))
    g = x.g if isinstance(case, str) else _rescale(x.g, case, None)
    gen = inputs.generator(3101)
    S0 = inputs.randn((B, H, D, D), gen, torch.float32, scale=0.05)
    if not isinstance(case, str):
        S0 = S0 * case  # a start state on the same scale as the values
    y, S = sala.lightning_prefill(x.q.cuda(), x.k.cuda(), v.cuda(), g.cuda(), S0.cuda().clone(),
                                  chunk=128, pos0=9)
    assert sala.get_device_error() == 0
    yr, Sr = oracle.lightning_recurrent(_np(x.q), _np(x.k), _np(v), _np(g), _np(S0), pos0=9)
    assert rel_err(_np(y), yr, True) <= TOL_BF16
    assert rel_err(_np(S), Sr, False) <= TOL_BF16


def test_lightning_segments_with_different_scales():
    """One head whose first third of v is scaled by 1e-6 and last third by 1e4: segments
    pick different exponents while the state carries across them."""
    B, T, H, D = 1, 128 * 12, 2, 128
    x = inputs.lightning_inputs(B, T, H, D, seed=3102)
    v = x.v.float().clone()
    v[:, :T // 3] *= 1e-6
    v[:, 2 * T // 3:] *= 1e4
    v = v.to(torch.bfloat16)
    y, S = sala.lightning_prefill(x.q.cuda(), x.k.cuda(), v.cuda(), x.g.cuda(), chunk=128)
    assert sala.get_device_error() == 0
    yr, Sr = oracle.lightning_recurrent(_np(x.q), _np(x.k), _np(v), _np(x.g))
    assert rel_err(_np(y), yr, True) <= TOL_BF16
    assert rel_err(_np(S), Sr, False) <= TOL_BF16
    # the rows before the large values are checked on their own scale as well
    r = slice(0, T // 3)
    assert rel_err(_np(y[:, r]), yr[:, r], True) <= TOL_BF16


@pytest.mark.parametrize("case", [1e-6, 1e3, "spike1e5"])
def test_lightning_state_call_scaled_v(case):
    """The state-only call (sequence-split Lightning) with far-from-unit v."""
    B, T, H, D = 1, 128 * 9 + 31, 3, 128
    x = inputs.lightning_inputs(B, T, H, D, seed=3103)
    v = _rescale(x.v, case, (0, 400, 2, 100))
    S = sala.lightning_state(x.k.cuda(), v.cuda(), None, chunk=128, pos0=4)
    assert sala.get_device_error() == 0
    _, Sr = oracle.lightning_recurrent(_np(x.k), _np(x.k), _np(v), pos0=4)
    assert rel_err(S.double().cpu().numpy(), Sr, False) <= TOL_BF16


@pytest.mark.parametrize("dtype,D,chunk", [(torch.float32, 64, 64), (torch.bfloat16, 128, 64)])
def test_lightning_cuda_core_scaled_v(dtype, D, chunk):
    """The CUDA-core kernel computes in fp32 throughout: v scaled by 1e-6 and 1e3."""
    B, T, H = 1, 300, 2
    x = inputs.lightning_inputs(B, T, H, D, seed=3104, dtype=dtype)
    for case in (1e-6, 1e3):
        v = _rescale(x.v, case, None)
        y, S = sala.lightning_prefill(x.q.cuda(), x.k.cuda(), v.cuda(), x.g.cuda(), chunk=chunk)
        yr, Sr = oracle.lightning_recurrent(_np(x.q), _np(x.k), _np(v), _np(x.g))
        bf = dtype == torch.bfloat16
        assert rel_err(_np(y), yr, bf) <= (TOL_BF16 if bf else TOL_F32)
        assert rel_err(_np(S), Sr, False) <= (TOL_BF16 if bf else TOL_F32)
    assert sala.get_device_error() == 0


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("D", [128, 64])
def test_sparse_attn_scaled_v(case, D):
    """Selection and block-sparse attention with far-from-unit v and gate; sampled rows."""
    T, Hq, Hkv = 64 * 40 + 9, 32, 2
    s = inputs.sparse_inputs(1, T, Hq, Hkv, D, seed=3200 + D, gate=True)
    v = _rescale(s.v, case, (0, 1000, 1, 7))
    g = s.g if isinstance(case, str) else _rescale(s.g, case, None)
    q, k = s.q.cuda(), s.k.cuda()
    idx = sala.sparse_select(q, k, topk=16)
    o = sala.sparse_attn(q, k, v.cuda(), idx, g.cuda())
    assert sala.get_device_error() == 0
    rows = np.unique(np.concatenate([np.arange(0, T, 7), np.arange(995, 1010), [T - 1]]))
    ref = oracle.attention(_np(s.q[:, rows]), _np(s.k), _np(v), _np(g[:, rows]),
                           idx=idx.cpu().numpy()[:, :, rows], rows=rows)
    assert rel_err(_np(o[:, rows]), ref, True) <= TOL_BF16


@pytest.mark.parametrize("case", CASES)
def test_sparse_decode_scaled_v(case):
    """Sparse-layer decode with far-from-unit v and gate: output against the oracle's
    attention over the GPU's selection."""
    B, Hq, Hkv, D, Tmax = 3, 32, 2, 128, 64 * 40
    gen = inputs.generator(3300)
    q = inputs.randn((B, Hq, D), gen)
    g = inputs.randn((B, Hq, D), gen)
    k = inputs.randn((B, Tmax, Hkv, D), gen)
    v = _rescale(inputs.randn((B, Tmax, Hkv, D), gen), case, (1, 64 * 38 + 2, 0, 3))
    if not isinstance(case, str):
        g = _rescale(g, case, None)
    kbar = sala.sparse_block_means(k.cuda())
    pos_l = [64 * 7 + 3, 64 * 38 + 20, Tmax - 1]
    idx = torch.empty((B, Hkv, 67), dtype=torch.int32, device=DEV)
    y = sala.sparse_decode(q.cuda(), k.cuda(), v.cuda(), kbar,
                           torch.tensor(pos_l, dtype=torch.int32, device=DEV), g.cuda(),
                           idx_out=idx)
    assert sala.get_device_error() == 0
    gi = idx.cpu().numpy()
    qn, kn, vn, gn = _np(q), _np(k), _np(v), _np(g)
    want = np.stack([oracle.attention(qn[b][None, None], kn[b:b + 1, :p + 1], vn[b:b + 1, :p + 1],
                                      gn[b][None, None], idx=gi[b][:, None, :], rows=[p])[0, 0]
                     for b, p in enumerate(pos_l)])
    assert rel_err(_np(y), want, True) <= TOL_BF16


def test_nonfinite_v_raises_range():
    """An infinite v raises SALA_ERR_RANGE through the device error word on every path
    that multiplies v on tensor cores (Lightning prefill, sparse attention, sparse decode)."""
    B, T, H, D = 1, 256, 1, 128
    x = inputs.lightning_inputs(B, T, H, D, seed=3400)
    v = x.v.clone()
    v[0, 17, 0, 5] = float("inf")
    sala.get_device_error()
    sala.lightning_prefill(x.q.cuda(), x.k.cuda(), v.cuda(), x.g.cuda(), chunk=128)
    assert sala.get_device_error() == SALA_ERR_RANGE
    assert sala.get_device_error() == 0
    for Dd in (128, 64):
        s = inputs.sparse_inputs(1, 300, 16, 1, Dd, seed=3401)
        vs = s.v.clone()
        vs[0, 10, 0, 3] = float("inf")
        dq, dk = s.q.cuda(), s.k.cuda()
        sala.sparse_attn(dq, dk, vs.cuda(), sala.sparse_select(dq, dk, topk=2))
        assert sala.get_device_error() == SALA_ERR_RANGE
        assert sala.get_device_error() == 0
    gen = inputs.generator(3402)
    q = inputs.randn((1, 16, 128), gen)
    k = inputs.randn((1, 128, 1, 128), gen)
    vd = inputs.randn((1, 128, 1, 128), gen)
    vd[0, 100, 0, 0] = float("inf")
    kbar = sala.sparse_block_means(k.cuda())
    sala.sparse_decode(q.cuda(), k.cuda(), vd.cuda(), kbar,
                       torch.tensor([127], dtype=torch.int32, device=DEV))
    assert sala.get_device_error() == SALA_ERR_RANGE
    assert sala.get_device_error() == 0
