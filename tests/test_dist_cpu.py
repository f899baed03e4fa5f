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


@pytest.mark.parametrize("lens", [(100, 157), (64, 64)])
def test_seqpar_host_logic_two_ranks(lens):
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_seqpar_worker, args=(world, _free_port(), list(lens), out), nprocs=world, join=True)
    for rank in range(world):
        dy, dS, scale = out[rank]
        assert dy <= 1e-10 and dS <= 1e-10 * max(1.0, scale)
