"""GPU parity: Lightning prefill and decode (libsala, through the C ABI) vs the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_long_lightning_b200 import inputs
from tests._parity import TOL_BF16, TOL_F32, raw_rel_err, rel_err

pytestmark = pytest.mark.gpu

sala = pytest.importorskip("sparse_attention_long_lightning_b200")
DEV = "cuda"


def _np(t):
    return t.detach().double().cpu().numpy()


def test_lightning_small_fp32_full():
    """Lightning, B1 H2 D64 T1024, fp32, chunk 64, seed 1001: every output and the state."""
    x = inputs.lightning_inputs(1, 1024, 2, 64, seed=1001, dtype=torch.float32)
    y, S = sala.lightning_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.g.cuda(), chunk=64)
    yr, Sr = oracle.lightning_recurrent(_np(x.q), _np(x.k), _np(x.v), _np(x.g))
    assert rel_err(_np(y), yr, False) <= TOL_F32
    assert rel_err(_np(S), Sr, False) <= TOL_F32


def _packed(B, T, H, D, dtype, seed):
    """q, k, v as non-contiguous views of one packed [B, T, 3, H, D] projection."""
    gen = inputs.generator(seed)
    qkv = inputs.randn((B, T, 3, H, D), gen, dtype)
    g = inputs.randn((B, T, H, D), gen, dtype)
    return qkv, g


@pytest.mark.parametrize("T,D,chunk,dtype", [
    (1, 128, 128, torch.bfloat16), (63, 128, 128, torch.bfloat16), (64, 128, 64, torch.bfloat16),
    (65, 128, 128, torch.bfloat16), (127, 128, 64, torch.bfloat16), (300, 128, 128, torch.bfloat16),
    (641, 128, 128, torch.bfloat16), (257, 64, 64, torch.bfloat16), (200, 128, 64, torch.float32),
    (129, 64, 128, torch.float32)])
def test_lightning_ragged_strided(T, D, chunk, dtype):
    """Ragged lengths, packed (strided) q/k/v, norm weights, a non-zero initial
    state and a position offset, B = 2, H = 3."""
    B, H = 2, 3
    qkv, g = _packed(B, T, H, D, dtype, seed=T * 7 + D)
    gen = inputs.generator(99)
    S0 = inputs.randn((B, H, D, D), gen, torch.float32, scale=0.05)
    qw = 1.0 + 0.1 * inputs.randn((D,), gen, torch.float32)
    kw = 1.0 + 0.1 * inputs.randn((D,), gen, torch.float32)
    dq = qkv.cuda()
    st = S0.cuda().clone()
    y, S = sala.lightning_prefill(dq[:, :, 0], dq[:, :, 1], dq[:, :, 2], g.cuda(), st,
                                  qw.cuda(), kw.cuda(), chunk=chunk, pos0=5)
    yr, Sr = oracle.lightning_recurrent(_np(qkv[:, :, 0]), _np(qkv[:, :, 1]), _np(qkv[:, :, 2]),
                                        _np(g), _np(S0), _np(qw), _np(kw), pos0=5)
    bf = dtype == torch.bfloat16
    tol = TOL_BF16 if bf else TOL_F32
    assert rel_err(_np(y), yr, bf) <= tol
    assert rel_err(_np(S), Sr, False) <= tol
    assert sala.get_device_error() == 0


def test_lightning_no_gate_zero_length():
    B, T, H, D = 1, 70, 2, 128
    x = inputs.lightning_inputs(B, T, H, D, seed=5, gate=False)
    y, S = sala.lightning_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), None, chunk=128)
    yr, Sr = oracle.lightning_recurrent(_np(x.q), _np(x.k), _np(x.v))
    assert rel_err(_np(y), yr, True) <= TOL_BF16
    # T = 0: the state passes through unchanged (or is zeroed when no state is given)
    st = S.clone()
    e = torch.empty((B, 0, H, D), dtype=torch.bfloat16, device=DEV)
    sala.lightning_prefill(e, e, e, None, st)
    torch.cuda.synchronize()
    assert torch.equal(st, S)


def test_lightning_segments_continue():
    """prefill(T1) then prefill(T2) from its state at pos0 = T1 equals the oracle on T1+T2."""
    B, T, H, D = 1, 700, 2, 128
    x = inputs.lightning_inputs(B, T, H, D, seed=11)
    dq, dk, dv, dg = (t.cuda() for t in (x.q, x.k, x.v, x.g))
    ya, S = sala.lightning_prefill(dq[:, :300], dk[:, :300], dv[:, :300], dg[:, :300])
    yb, S = sala.lightning_prefill(dq[:, 300:], dk[:, 300:], dv[:, 300:], dg[:, 300:], S,
                                   pos0=300)
    yr, Sr = oracle.lightning_recurrent(_np(x.q), _np(x.k), _np(x.v), _np(x.g))
    assert rel_err(_np(torch.cat([ya, yb], 1)), yr, True) <= TOL_BF16
    assert rel_err(_np(S), Sr, False) <= TOL_BF16


def test_lightning_32k_full_size_sampled_heads():
    """Lightning prefill B1 H32 D128 T32768 bf16, chunk 128, seed 1002 (the launch
    the benchmark times): four heads compared on every row, plus their final state."""
    B, T, H, D = 1, 32768, 32, 128
    x = inputs.lightning_inputs(B, T, H, D, seed=1002, device=DEV)
    y, S = sala.lightning_prefill(x.q, x.k, x.v, x.g, chunk=128)
    heads = [0, 7, 19, 31]
    yr, Sr = oracle.lightning_recurrent(*(_np(t[:, :, heads]) for t in (x.q, x.k, x.v, x.g)))
    e_y = rel_err(_np(y[:, :, heads]), yr, True)
    e_s = rel_err(_np(S[:, heads]), Sr, False)
    print(f"32k: y {e_y:.3e} (raw {raw_rel_err(_np(y[:, :, heads]), yr):.3e}) S {e_s:.3e}")
    assert e_y <= TOL_BF16 and e_s <= TOL_BF16
    assert sala.get_device_error() == 0


def test_lightning_1m_full_size_sampled_head():
    """One Lightning layer of the 1M-token hybrid stack: B1 H32 D128 T1048576 bf16,
    chunk 128 (seed 1012).  One head is compared on 4096 spread rows plus the last 128,
    and its final state, against the full 1M-token recurrence."""
    B, T, H, D = 1, 1 << 20, 32, 128
    x = inputs.lightning_inputs(B, T, H, D, seed=1012, device=DEV)
    y, S = sala.lightning_prefill(x.q, x.k, x.v, x.g, chunk=128)
    head = 13
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([rng.choice(T - 128, size=4096, replace=False),
                                     np.arange(T - 128, T)]))
    yr, Sr = oracle.lightning_recurrent(*(_np(t[:, :, [head]]) for t in (x.q, x.k, x.v, x.g)),
                                        rows=rows)
    e_y = rel_err(_np(y[:, rows][:, :, [head]]), yr, True)
    e_s = rel_err(_np(S[:, [head]]), Sr, False)
    print(f"1m: y {e_y:.3e} S {e_s:.3e}")
    assert e_y <= TOL_BF16 and e_s <= TOL_BF16
    assert sala.get_device_error() == 0


@pytest.mark.parametrize("D,dtype", [(128, torch.bfloat16), (64, torch.float32)])
def test_decode_steps(D, dtype):
    B, H, steps = 3, 4, 5
    gen = inputs.generator(1234)
    S0 = inputs.randn((B, H, D, D), gen, torch.float32, scale=1.0 / 64)
    qw = 1.0 + 0.1 * inputs.randn((D,), gen, torch.float32)
    st = S0.cuda().clone()
    Sref = _np(S0)
    for s in range(steps):
        q, k, v, g = inputs.decode_tokens(B, H, D, seed=77, step=s, dtype=dtype)
        pos = torch.tensor([s, 1000 + s, 123456 + s], dtype=torch.int32)
        y = sala.lightning_decode(q.cuda(), k.cuda(), v.cuda(), g.cuda(), st, pos.cuda(),
                                  qw.cuda(), None)
        yr, Sref = oracle.lightning_decode(_np(q), _np(k), _np(v), _np(g), Sref, pos.numpy(),
                                           _np(qw), None)
        bf = dtype == torch.bfloat16
        tol = TOL_BF16 if bf else TOL_F32
        assert rel_err(_np(y), yr, bf) <= tol
    assert rel_err(_np(st), Sref, False) <= (TOL_BF16 if dtype == torch.bfloat16 else TOL_F32)


def test_decode_full_size_256_steps():
    """The whole decode workload: B64 H32 D128, state N(0,1)/64 (seed 1003), 256 steps of
    one new token (step s from seed 1003*1000+1+s, position s), the state updated in place
    on the GPU.  Every step's output, and the state after steps 1, 64, 128 and 256, against
    the fp64 recurrence, so drift over the in-place updates would show."""
    B, H, D, steps = 64, 32, 128, 256
    S0 = inputs.decode_state(B, H, D, seed=1003, device=DEV)
    st = S0.clone()
    Sref = _np(S0)
    worst = 0.0
    for s in range(steps):
        q, k, v, g = inputs.decode_tokens(B, H, D, seed=1003, step=s, device=DEV)
        pos = torch.full((B,), s, dtype=torch.int32, device=DEV)
        y = sala.lightning_decode(q, k, v, g, st, pos)
        yr, Sref = oracle.lightning_decode(_np(q), _np(k), _np(v), _np(g), Sref, np.full(B, s),
                                           inplace=True)
        e = rel_err(_np(y), yr, True)
        worst = max(worst, e)
        assert e <= TOL_BF16, (s, e)
        if s + 1 in (1, 64, 128, 256):
            assert rel_err(_np(st), Sref, False) <= TOL_BF16, s
    print(f"decode 256 steps: worst output error {worst:.3e}, final state "
          f"{rel_err(_np(st), Sref, False):.3e}")
    assert sala.get_device_error() == 0


def test_decode_continues_prefill():
    """GPU prefill(T) then GPU decode at pos T matches oracle prefill(T+1) row T."""
    B, T, H, D = 1, 200, 2, 128
    x = inputs.lightning_inputs(B, T + 1, H, D, seed=21)
    dq, dk, dv, dg = (t.cuda() for t in (x.q, x.k, x.v, x.g))
    _, S = sala.lightning_prefill(dq[:, :T], dk[:, :T], dv[:, :T], dg[:, :T])
    pos = torch.full((B,), T, dtype=torch.int32, device=DEV)
    y = sala.lightning_decode(dq[:, T], dk[:, T], dv[:, T], dg[:, T], S, pos)
    yr, _ = oracle.lightning_recurrent(*(_np(t) for t in (x.q, x.k, x.v, x.g)), rows=[T])
    assert rel_err(_np(y), yr[:, 0], True) <= TOL_BF16


def test_lightning_large_state_rescaling():
    """Keys nearly constant and values ~500: the state grows past the fp16 range
    within one chunk, so the tensor-core path must rescale its fp16 copy of S by
    powers of two; the result must still match the oracle."""
    B, T, H, D = 1, 1000, 2, 128
    gen = inputs.generator(4242)
    base = inputs.randn((1, 1, H, D), gen, torch.float32)
    k = (base + 0.01 * inputs.randn((B, T, H, D), gen, torch.float32)).to(torch.bfloat16)
    q = inputs.randn((B, T, H, D), gen)
    v = (500.0 + inputs.randn((B, T, H, D), gen, torch.float32)).to(torch.bfloat16)
    g = inputs.randn((B, T, H, D), gen)
    y, S = sala.lightning_prefill(q.cuda(), k.cuda(), v.cuda(), g.cuda(), chunk=128)
    yr, Sr = oracle.lightning_recurrent(_np(q), _np(k), _np(v), _np(g))
    assert float(np.abs(Sr).max()) > 65504.0  # the state really left the fp16 range
    assert rel_err(_np(y), yr, True) <= TOL_BF16
    assert rel_err(_np(S), Sr, False) <= TOL_BF16
    assert sala.get_device_error() == 0


# ---------------------------------------------------------------------------------------
# Sequence split across devices: segment states (sala_lightning_state), their prefix
# (sala_state_prefix_sum) and the segment prefills, run here rank after rank on one GPU.
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("D,dtype,chunk", [(128, torch.bfloat16, 128), (64, torch.float32, 64),
                                           (128, torch.bfloat16, 64)])
def test_lightning_state_matches_prefill_final_state(D, dtype, chunk):
    """The state-only call gives the prefill's final state (zero start and a given start)."""
    B, T, H = 1, 64 * 21 + 5, 4
    x = inputs.lightning_inputs(B, T, H, D, seed=61, dtype=dtype, device=DEV)
    _, S_pf = sala.lightning_prefill(x.q, x.k, x.v, x.g, None, chunk=chunk, pos0=7)
    S = sala.lightning_state(x.k, x.v, None, chunk=chunk, pos0=7)
    tol = TOL_F32 if dtype == torch.float32 else 1e-6
    assert raw_rel_err(S.cpu().numpy(), S_pf.cpu().numpy()) <= tol
    S0 = torch.randn((B, H, D, D), generator=torch.Generator(device=DEV).manual_seed(3),
                     device=DEV) * 0.05
    _, S_pf0 = sala.lightning_prefill(x.q, x.k, x.v, x.g, S0.clone(), chunk=chunk, pos0=7)
    S1 = sala.lightning_state(x.k, x.v, S0.clone(), chunk=chunk, pos0=7)
    assert raw_rel_err(S1.cpu().numpy(), S_pf0.cpu().numpy()) <= tol
    _, S_or = oracle.lightning_recurrent(_np(x.k), _np(x.k), _np(x.v), pos0=7)
    assert raw_rel_err(S.cpu().numpy(), S_or) <= (TOL_F32 if dtype == torch.float32 else TOL_BF16)


def test_lightning_sequence_split_three_segments():
    """Three uneven segments processed as three ranks would: states, prefix, segment
    prefills.  Outputs and final state agree with one prefill of the whole sequence and
    with the oracle."""
    B, H, D = 1, 8, 128
    lens = [1000, 1024 + 77, 930]
    T = sum(lens)
    x = inputs.lightning_inputs(B, T, H, D, seed=62, device=DEV)
    S_init = torch.randn((B, H, D, D), generator=torch.Generator(device=DEV).manual_seed(4),
                         device=DEV) * 0.02
    y_full, S_full = sala.lightning_prefill(x.q, x.k, x.v, x.g, S_init.clone(), pos0=11)
    offs = [0, lens[0], lens[0] + lens[1]]
    seg = lambda t, r: t[:, offs[r]:offs[r] + lens[r]]
    dS = torch.stack([sala.lightning_state(seg(x.k, r), seg(x.v, r), None, pos0=11 + offs[r])
                      for r in range(3)])
    ys = []
    for r in range(3):
        S0 = sala.state_prefix_sum(dS, r, S_init.clone(), accumulate=True)
        y, S_end = sala.lightning_prefill(seg(x.q, r), seg(x.k, r), seg(x.v, r), seg(x.g, r), S0,
                                          pos0=11 + offs[r])
        ys.append(y)
    y_split = torch.cat(ys, dim=1)
    assert sala.get_device_error() == 0
    from tests._parity import rel_err_bf16_pair
    assert rel_err_bf16_pair(_np(y_split), _np(y_full)) <= TOL_BF16
    # segments start off the 128-token chunk grid, so a token's RoPE angle is formed from a
    # different chunk base (and rounds differently before the fp16 operand cast): the two
    # final states agree to ~1e-4, both within the oracle tolerance checked below
    assert raw_rel_err(S_end.cpu().numpy(), S_full.cpu().numpy()) <= 1e-3
    y_or, S_or = oracle.lightning_recurrent(_np(x.q), _np(x.k), _np(x.v), _np(x.g),
                                            S_init.double().cpu().numpy(), pos0=11)
    assert rel_err(_np(y_split), y_or, bf16_out=True) <= TOL_BF16
    assert raw_rel_err(S_end.cpu().numpy(), S_or) <= TOL_BF16


def test_lightning_seqpar_single_rank_group():
    """The public sequence-parallel call on a one-rank NCCL group is the plain prefill."""
    import os
    import socket

    import torch.distributed as dist

    from sparse_attention_long_lightning_b200.seqpar import lightning_prefill_seqpar
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ["MASTER_ADDR"], os.environ["MASTER_PORT"] = "127.0.0.1", str(port)
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        x = inputs.lightning_inputs(1, 777, 4, 128, seed=63, device=DEV)
        y, S = lightning_prefill_seqpar(x.q, x.k, x.v, x.g, pos0=3)
        y_ref, S_ref = sala.lightning_prefill(x.q, x.k, x.v, x.g, None, pos0=3)
        assert torch.equal(y, y_ref)
        assert raw_rel_err(S.cpu().numpy(), S_ref.cpu().numpy()) <= 1e-6
    finally:
        dist.destroy_process_group()
