"""The allocation-free Lightning prefill entry point.

Some callers of this library cannot hand it a workspace: a host framework that
owns every device allocation and gives its plugins no allocator, or a serving
loop whose memory pool is frozen after start-up.  sala_lightning_prefill_noalloc
serves them from a fixed scratch array inside the library.  These tests call it
through the C ABI and compare it with the fp64 oracle (and with the regular entry
point), twice in a row (the second call reuses the scratch the first one left
behind), including a call that fills the scratch.  The file is named so that
pytest collects it last.
"""
import pytest
import torch

import oracle
from sparse_attention_long_lightning_b200 import inputs
from tests._parity import TOL_BF16, rel_err, rel_err_bf16_pair

pytestmark = pytest.mark.gpu

sala = pytest.importorskip("sparse_attention_long_lightning_b200")


def _np(t):
    return t.detach().double().cpu().numpy()


def _check_twice(B, T, H, seed):
    """Two calls in a row (the second reuses what the first left in the scratch), each
    against the fp64 oracle; the regular entry point is compared as well."""
    D = 128
    x = inputs.lightning_inputs(B, T, H, D, seed=seed, device="cuda")
    gen = inputs.generator(seed + 1)
    S0 = inputs.randn((B, H, D, D), gen, torch.float32, scale=0.05).cuda()
    yr, Sr = oracle.lightning_recurrent(_np(x.q), _np(x.k), _np(x.v), _np(x.g), _np(S0), pos0=3)
    ref_o, ref_S = sala.lightning_prefill(x.q, x.k, x.v, x.g, S0.clone(), chunk=128, pos0=3)
    for _ in range(2):
        out = torch.empty_like(x.q)
        state = S0.clone()
        sala.lightning_prefill_noalloc(x.q, x.k, x.v, x.g, state, out, chunk=128, pos0=3)
        torch.cuda.synchronize()
        assert rel_err(_np(out), yr, True) <= TOL_BF16
        assert rel_err(_np(state), Sr, False) <= TOL_BF16
        # the regular entry point runs more segments, so each output rounds to bf16 from a
        # slightly different fp32 value: half an ulp of each side is allowed
        assert rel_err_bf16_pair(_np(out), _np(ref_o)) <= TOL_BF16
        assert rel_err(_np(state), _np(ref_S), False) <= TOL_BF16
    assert sala.get_device_error() == 0


def test_noalloc_matches_oracle_twice():
    _check_twice(1, 8192 + 77, 32, seed=2024)


def test_noalloc_at_scratch_capacity():
    """B*H = 256 heads fill the scratch: one segment per head (the regular entry point
    would split each head into several)."""
    _check_twice(2, 300, 128, seed=2025)


def test_noalloc_rejects_too_many_heads():
    """B*H above the scratch capacity (256 segment states) is refused before any launch."""
    B, T, H, D = 2, 128, 160, 128
    x = inputs.lightning_inputs(B, T, H, D, seed=5, device="cuda")
    out = torch.empty_like(x.q)
    state = torch.zeros((B, H, D, D), dtype=torch.float32, device="cuda")
    with pytest.raises(sala.SalaError) as exc:
        sala.lightning_prefill_noalloc(x.q, x.k, x.v, x.g, state, out, init_zero=True)
    assert exc.value.status == 5
