"""GPU: a hybrid decode step (one Lightning layer, one sparse layer) captured once as a
CUDA graph and replayed step after step gives the same outputs and the same in-place
state updates (Lightning state, block-mean cache) as eager calls, bit for bit (the
decode kernels' parity with the oracle is checked in test_gpu_lightning.py and
test_gpu_sparse_decode.py)."""
import pytest
import torch

from sparse_attention_long_lightning_b200 import inputs

pytestmark = pytest.mark.gpu

sala = pytest.importorskip("sparse_attention_long_lightning_b200")
DEV = "cuda"


def test_decode_step_graph_matches_eager():
    from sparse_attention_long_lightning_b200.graphs import StaticStep

    B, H, Hkv, D, Tmax, T0, steps = 4, 32, 2, 128, 64 * 24, 64 * 20 + 60, 9
    S0 = inputs.decode_state(B, H, D, seed=71, device=DEV)
    gen = inputs.generator(72, DEV)
    kc = inputs.randn((B, Tmax, Hkv, D), gen, device=DEV)
    vc = inputs.randn((B, Tmax, Hkv, D), gen, device=DEV)
    kbar0 = torch.zeros((B, Tmax // 64, Hkv, D), dtype=torch.float32, device=DEV)
    sala.sparse_block_means(kc[:, :T0], kbar0)
    toks = [inputs.decode_tokens(B, H, D, seed=73, step=s, device=DEV) for s in range(steps)]
    qs = [inputs.decode_tokens(B, H, D, seed=74, step=s, device=DEV)[0] for s in range(steps)]

    # static buffers read by the captured step
    st = {"q": torch.empty_like(toks[0][0]), "k": torch.empty_like(toks[0][1]),
          "v": torch.empty_like(toks[0][2]), "g": torch.empty_like(toks[0][3]),
          "qs": torch.empty_like(qs[0]), "pos": torch.full((B,), T0, dtype=torch.int32,
                                                            device=DEV)}
    S, kbar = S0.clone(), kbar0.clone()
    out_l, out_s = torch.empty_like(st["q"]), torch.empty_like(st["qs"])
    ws = torch.empty(sala.sparse_decode_workspace(B, Tmax, H, Hkv, D, 67), dtype=torch.uint8,
                     device=DEV)

    def step():
        sala.lightning_decode(st["q"], st["k"], st["v"], st["g"], S, st["pos"], out=out_l)
        sala.sparse_decode(st["qs"], kc, vc, kbar, st["pos"], st["g"], out=out_s, workspace=ws)

    def restore():
        S.copy_(S0)
        kbar.copy_(kbar0)

    q0, k0, v0, g0 = toks[0]
    for name, val in (("q", q0), ("k", k0), ("v", v0), ("g", g0), ("qs", qs[0])):
        st[name].copy_(val)  # the eager warm-up reads real tokens
    graph_step = StaticStep(step, st, restore=restore)
    torch.cuda.synchronize()

    # eager reference on its own copies of the state
    S_e, kbar_e = S0.clone(), kbar0.clone()
    for s in range(steps):
        q, k, v, g = toks[s]
        pos = torch.full((B,), T0 + s, dtype=torch.int32, device=DEV)
        graph_step.set(q=q, k=k, v=v, g=g, qs=qs[s], pos=pos)
        graph_step.replay()
        y_l = sala.lightning_decode(q, k, v, g, S_e, pos)
        y_s = sala.sparse_decode(qs[s], kc, vc, kbar_e, pos, g)
        torch.cuda.synchronize()
        assert torch.equal(out_l, y_l), s
        assert torch.equal(out_s, y_s), s
    assert torch.equal(S, S_e)
    assert torch.equal(kbar, kbar_e)  # the steps crossed a block end: the cache was updated
    assert not torch.equal(kbar, kbar0)
    assert sala.get_device_error() == 0
