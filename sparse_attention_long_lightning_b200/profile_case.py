"""Run one hot-path operation at a chosen size, for profiler captures and quick timing.

    python -m sparse_attention_long_lightning_b200.profile_case --op attn --T 16384 --iters 3

Ops: lightning (prefill, B1 H32 D128 bf16 chunk 128), lightning_prepared (the same on
prepared fp16 q/k operands), proj (the fused input projection of a Lightning layer, T
tokens x hidden -> 4 x 32 heads of 128), decode (B64 H32 D128 bf16),
select / attn (B1 Hq32 Hkv2 D128 bf16, top-64 + 1 + 2), sparse_decode (B sequences,
Hq32 Hkv2 D128 bf16, KV caches of T tokens, one step at positions near the end).
Prints the mean CUDA-event time per call.
"""
from __future__ import annotations

import argparse

import torch

import sparse_attention_long_lightning_b200 as sala
from sparse_attention_long_lightning_b200 import inputs


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", required=True, choices=["lightning", "decode", "select", "attn",
                                                       "sparse_decode", "select_hsm", "proj",
                                                       "lightning_prepared"])
    ap.add_argument("--hidden", type=int, default=4096, help="hidden size for proj")
    ap.add_argument("--T", type=int, default=16384)
    ap.add_argument("--B", type=int, default=64, help="batch for decode")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=1)
    a = ap.parse_args()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if a.op == "lightning":
        x = inputs.lightning_inputs(1, a.T, 32, 128, seed=1002, device=dev)
        o = torch.empty_like(x.q)
        ws = torch.empty(max(1, sala.lightning_prefill_workspace(1, a.T, 32, 128, 128)),
                         dtype=torch.uint8, device=dev)
        fn = lambda: sala.lightning_prefill(x.q, x.k, x.v, x.g, None, chunk=128, out=o,
                                            workspace=ws)
    elif a.op == "lightning_prepared":
        gen = inputs.generator(1002, dev)
        qh = inputs.randn((1, a.T, 32, 128), gen, torch.float16, dev)
        kh = inputs.randn((1, a.T, 32, 128), gen, torch.float16, dev)
        v = inputs.randn((1, a.T, 32, 128), gen, device=dev)
        gate = inputs.randn((1, a.T, 32, 128), gen, device=dev).sigmoid().to(torch.float16)
        o = torch.empty_like(v)
        ws = torch.empty(max(1, sala.lightning_prefill_workspace(1, a.T, 32, 128, 128)),
                         dtype=torch.uint8, device=dev)
        fn = lambda: sala.lightning_prefill_prepared(qh, kh, v, gate, None, out=o, workspace=ws)
    elif a.op == "proj":
        gen = inputs.generator(1008, dev)
        x = inputs.randn((1, a.T, a.hidden), gen, device=dev)
        w = inputs.randn((4 * 32 * 128, a.hidden), gen, device=dev, scale=a.hidden ** -0.5)
        outs = sala.lightning_projection(x, w, heads=32, head_dim=128)
        fn = lambda: sala.lightning_projection(x, w, heads=32, head_dim=128, out=outs)
        print(f"proj: {2.0 * a.T * a.hidden * 4 * 32 * 128 / 1e12:.3f} TFLOP per call")
    elif a.op == "decode":
        S = inputs.decode_state(a.B, 32, 128, seed=1003, device=dev)
        q, k, v, g = inputs.decode_tokens(a.B, 32, 128, seed=1003, step=0, device=dev)
        pos = torch.zeros(a.B, dtype=torch.int32, device=dev)
        o = torch.empty_like(q)
        fn = lambda: sala.lightning_decode(q, k, v, g, S, pos, out=o)
    elif a.op == "sparse_decode":
        B, Tmax = a.B, a.T
        gen = inputs.generator(1006, dev)
        k = inputs.randn((B, Tmax, 2, 128), gen, device=dev)
        v = inputs.randn((B, Tmax, 2, 128), gen, device=dev)
        q = inputs.randn((B, 32, 128), gen, device=dev)
        g = inputs.randn((B, 32, 128), gen, device=dev)
        kbar = sala.sparse_block_means(k)
        pos = torch.tensor([Tmax - 1 - 13 * b for b in range(B)], dtype=torch.int32, device=dev)
        ws = torch.empty(sala.sparse_decode_workspace(B, Tmax, 32, 2, 128, 67), dtype=torch.uint8,
                         device=dev)
        o = torch.empty_like(q)
        fn = lambda: sala.sparse_decode(q, k, v, kbar, pos, g, out=o, workspace=ws)
        cand = sum(max(0, (Tmax - 1 - 13 * b) // 64 - 2) for b in range(B))
        nbytes = cand * 2 * 128 * 4 + B * 2 * 67 * 64 * 128 * 2 * 2 + 3 * B * 32 * 128 * 2
        print(f"sparse_decode: algorithmic bytes per step {nbytes / 1e6:.1f} MB "
              f"(block means {cand * 2 * 128 * 4 / 1e6:.1f} MB, K/V blocks "
              f"{B * 2 * 67 * 64 * 128 * 4 / 1e6:.1f} MB)")
    else:
        s = inputs.sparse_inputs(1, a.T, 32, 2, 128, seed=1004, device=dev, gate=True)
        idx = sala.sparse_select(s.q, s.k)
        ws = torch.empty(max(sala.sparse_select_workspace(1, a.T, 32, 2, 128, 64, 64),
                             sala.sparse_attn_workspace(1, a.T, 2, 128)), dtype=torch.uint8,
                         device=dev)
        o = torch.empty_like(s.q)
        if a.op == "select":
            fn = lambda: sala.sparse_select(s.q, s.k, out=idx, workspace=ws)
        elif a.op == "select_hsm":
            wsh = torch.empty(sala.sparse_select_head_softmax_workspace(1, a.T, 32, 2, 128),
                              dtype=torch.uint8, device=dev)
            fn = lambda: sala.sparse_select(s.q, s.k, out=idx, workspace=wsh, score="head_softmax")
            # per-head scores: 2 passes x (query heads x candidate pairs) x D multiply-adds
            pairs = sum(max(0, t // 64 - 2) for t in range(a.T)) * 32
            print(f"select_hsm: {pairs * 128 * 2 / 1e12:.3f} T multiply-adds per call "
                  f"(two passes over {pairs / 1e9:.2f} G query-head x candidate pairs)")
        else:
            fn = lambda: sala.sparse_attn(s.q, s.k, s.v, idx, s.g, out=o, workspace=ws)
    for _ in range(a.warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    err = sala.get_device_error()
    print(f"{a.op} T={a.T}: {e0.elapsed_time(e1) / a.iters:.3f} ms/call, device_error={err}")
    return 1 if err else 0


if __name__ == "__main__":
    raise SystemExit(main())
