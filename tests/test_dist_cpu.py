"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the job's step time
is the maximum over ranks and the reported throughput is weak-scaling (every rank
processes its own sequence)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        local = [0.125, 0.25][rank]
        sec = bench.max_over_ranks(dist, local, torch.device("cpu"))
        out[rank] = (sec, bench.weak_scaling_value(world, 131072, sec))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_step_time_is_max_over_ranks():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        sec, value = out[rank]
        assert sec == 0.25
        assert value == pytest.approx(2 * 131072 / 0.25)


def test_single_process_passthrough():
    import bench
    assert bench.max_over_ranks(None, 0.5, torch.device("cpu")) == 0.5
    assert bench.weak_scaling_value(1, 1000, 0.5) == 2000


def test_bench_gpus_flag_launches_ranks(monkeypatch):
    """`--gpus N` outside torchrun starts N ranks through torch.distributed.run on
    127.0.0.1; inside torchrun a WORLD_SIZE that differs from N is an error; N = 1 runs
    in this process."""
    import argparse

    import bench
    calls = []
    monkeypatch.setattr(bench.subprocess, "call", lambda cmd: calls.append(cmd) or 0)
    monkeypatch.setattr(bench.sys, "argv", ["bench.py", "--gpus", "4", "--steps", "3"])
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    assert bench.launch_ranks(argparse.Namespace(gpus=4)) == 0
    cmd = calls[0]
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "127.0.0.1" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "3"]
    assert bench.launch_ranks(argparse.Namespace(gpus=1)) is None
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.launch_ranks(argparse.Namespace(gpus=4)) == 2
    assert bench.launch_ranks(argparse.Namespace(gpus=2)) is None


def test_bench_reference_sample_is_labelled(monkeypatch):
    """The oracle sample used by both CPU legs states its scale factors."""
    import bench
    monkeypatch.setitem(bench.ORACLE_SAMPLE, "light_tokens", 64)
    monkeypatch.setitem(bench.ORACLE_SAMPLE, "sparse_rows", 4)
    smp = bench.OracleSample(4096)
    info = smp.info()
    assert info["extrapolated"] is True and info["kind"] == "oracle"
    assert info["factor"]["lightning"] == 6 * 32 * 4096 / (16 * 64)
    assert info["factor"]["sparse"] == 2 * 4096 / 4
    sample_s, full_s = smp.time()
    assert 0 < sample_s < full_s


def test_bench_build_digest_is_stable():
    import bench
    a, b = bench.source_digest(), bench.source_digest()
    assert a == b and len(a) == 12 and int(a, 16) >= 0


# ---------------------------------------------------------------------------------------
# Sequence-parallel Lightning prefill: the multi-rank host logic (segment offsets, the
# all-gather of segment states in rank order, the prefix) on CPU ranks, with the fp64
# oracle standing in for the kernels.  The GPU kernels of the same steps are checked in
# tests/test_gpu_lightning.py.
# ---------------------------------------------------------------------------------------

def _seqpar_worker(rank, world, port, lens, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta

    import numpy as np

    import oracle
    from sparse_attention_long_lightning_b200.seqpar import seqpar_prefill
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        rng = np.random.default_rng(99)
        T, H, D = sum(lens), 2, 16
        q, k, v, g = (rng.standard_normal((1, T, H, D)) for _ in range(4))
        S_init = rng.standard_normal((1, H, D, D)) * 0.1
        offsets = [0] + list(np.cumsum(lens)[:-1])
        a, b = offsets[rank], offsets[rank] + lens[rank]

        def state_fn(kk, vv, pos):  # contribution of the segment alone
            _, S = oracle.lightning_recurrent(kk, kk, vv, pos0=pos)
            return torch.from_numpy(S)

        def gather_states(dS):
            parts = [torch.empty_like(dS) for _ in range(world)]
            dist.all_gather(parts, dS)
            return torch.stack(parts)

        def prefix_fn(gathered, r, S0):
            return S0 + gathered[:r].sum(0).numpy()

        def prefill_fn(qq, kk, vv, gg, S0, pos):
            return oracle.lightning_recurrent(qq, kk, vv, gg, S0, pos0=pos)

        y, S_end = seqpar_prefill(q[:, a:b], k[:, a:b], v[:, a:b], g[:, a:b], S_init, rank=rank,
                                  offsets=offsets, pos0=5, gather_states=gather_states,
                                  state_fn=state_fn, prefix_fn=prefix_fn, prefill_fn=prefill_fn)
        y_full, S_full = oracle.lightning_recurrent(q, k, v, g, S_init, pos0=5)
        out[rank] = (float(np.abs(y - y_full[:, a:b]).max()),
                     float(np.abs(S_end - oracle.lightning_recurrent(
                         q[:, :b], k[:, :b], v[:, :b], g[:, :b], S_init, pos0=5)[1]).max()),
                     float(np.abs(S_full).max()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lens", [(100, 157), (64, 64), (37, 128, 90)])
def test_seqpar_host_logic_multi_rank(lens):
    world = len(lens)
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_seqpar_worker, args=(world, _free_port(), list(lens), out), nprocs=world, join=True)
    for rank in range(world):
        dy, dS, scale = out[rank]
        assert dy <= 1e-10 and dS <= 1e-10 * max(1.0, scale)


# ---------------------------------------------------------------------------------------
# KV-head-parallel sparse layer: each rank selects and attends on its own KV heads and
# their query groups; the all-gathered output must equal the full layer exactly (the
# per-KV-head computations are independent).  fp64 oracle standing in for the kernels.
# ---------------------------------------------------------------------------------------

def _headpar_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta

    import numpy as np

    import oracle
    from sparse_attention_long_lightning_b200.seqpar import sparse_layer_headpar
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        rng = np.random.default_rng(123)
        T, Hq, Hkv, D, topk = 64 * 12 + 5, 8, 4, 16, 3
        q, g = (torch.from_numpy(rng.standard_normal((1, T, Hq, D))) for _ in range(2))
        k, v = (torch.from_numpy(rng.standard_normal((1, T, Hkv, D))) for _ in range(2))

        def select_fn(qq, kk):
            return oracle.sparse_select(qq.numpy(), kk.numpy(), topk=topk)[0]

        def attn_fn(qq, kk, vv, idx, gg):
            return torch.from_numpy(oracle.attention(qq.numpy(), kk.numpy(), vv.numpy(),
                                                     gg.numpy(), idx=idx))

        def gather_fn(o_r):
            parts = [torch.empty_like(o_r) for _ in range(world)]
            dist.all_gather(parts, o_r.contiguous())
            return parts

        y = sparse_layer_headpar(q, k, v, g, rank=rank, world=world, select_fn=select_fn,
                                 attn_fn=attn_fn, gather_fn=gather_fn)
        idx_full = select_fn(q, k)
        y_full = attn_fn(q, k, v, idx_full, g)
        out[rank] = (tuple(y.shape), float((y - y_full).abs().max()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_sparse_kvhead_parallel_ranks(world):
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_headpar_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        shape, err = out[rank]
        assert shape == (1, 64 * 12 + 5, 8, 16)
        assert err == 0.0


def test_kvhead_ranges_cover_all_heads():
    from sparse_attention_long_lightning_b200.seqpar import kvhead_range
    for Hkv in (1, 2, 3, 8):
        for world in range(1, Hkv + 1):
            spans = [kvhead_range(Hkv, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == Hkv
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            assert all(hi > lo for lo, hi in spans)
    with pytest.raises(ValueError):
        kvhead_range(2, 0, 3)


# ---------------------------------------------------------------------------------------
# Query-range-parallel sparse layer: each rank holds a contiguous token segment, gathers
# the whole sequence's k and v, and selects / attends for its own rows at their positions.
# fp64 oracle (row windows) standing in for the kernels; the gathered output must equal
# the whole-sequence layer exactly (rows are independent).
# ---------------------------------------------------------------------------------------

def _qrange_worker(rank, world, port, lens, B, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta

    import numpy as np

    import oracle
    from sparse_attention_long_lightning_b200.seqpar import (gather_token_segments,
                                                             segment_offsets,
                                                             sparse_layer_qrange)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        rng = np.random.default_rng(321)
        T, Hq, Hkv, D, topk = sum(lens), 4, 2, 16, 3
        q, g = (torch.from_numpy(rng.standard_normal((B, T, Hq, D))) for _ in range(2))
        k, v = (torch.from_numpy(rng.standard_normal((B, T, Hkv, D))) for _ in range(2))
        offs = segment_offsets(lens)
        lo, hi = offs[rank], offs[rank] + lens[rank]
        seg = lambda x: x[:, lo:hi].contiguous()  # this rank's tokens

        def gather_kv(kk, vv):
            return gather_token_segments(kk, lens), gather_token_segments(vv, lens)

        def select_fn(qq, K, p):
            rows = list(range(p, p + qq.shape[1]))
            return oracle.sparse_select(qq.numpy(), K.numpy(), topk=topk, rows=rows, T=K.shape[1])[0]

        def attn_fn(qq, K, V, idx, gg, p):
            rows = list(range(p, p + qq.shape[1]))
            return torch.from_numpy(oracle.attention(qq.numpy(), K.numpy(), V.numpy(), gg.numpy(),
                                                     idx=idx, rows=rows))

        y = sparse_layer_qrange(seg(q), seg(k), seg(v), seg(g), rank=rank, offsets=offs,
                                gather_kv=gather_kv, select_fn=select_fn, attn_fn=attn_fn,
                                gather_fn=lambda o: gather_token_segments(o, lens))
        idx_full = oracle.sparse_select(q.numpy(), k.numpy(), topk=topk)[0]
        y_full = torch.from_numpy(oracle.attention(q.numpy(), k.numpy(), v.numpy(), g.numpy(),
                                                   idx=idx_full))
        out[rank] = (tuple(y.shape), float((y - y_full).abs().max()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lens,B", [
    ((400, 400), 1),             # equal segments: the in-place all-gather
    ((300, 517, 40), 1),         # three uneven segments, one shorter than a block
    ((64 * 5 + 3, 64 * 4), 2),   # two sequences per rank
])
def test_sparse_query_parallel_ranks(lens, B):
    world = len(lens)
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_qrange_worker, args=(world, _free_port(), list(lens), B, out), nprocs=world,
             join=True)
    for rank in range(world):
        shape, err = out[rank]
        assert shape == (B, sum(lens), 4, 16)
        assert err == 0.0


def test_segment_offsets():
    from sparse_attention_long_lightning_b200.seqpar import segment_offsets
    assert segment_offsets([3, 0, 5]) == [0, 3, 3]
    assert segment_offsets([]) == []
    with pytest.raises(ValueError):
        segment_offsets([2, -1])
