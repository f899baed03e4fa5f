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
