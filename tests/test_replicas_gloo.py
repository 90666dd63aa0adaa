"""The multi-GPU host path of bench.py (replicas, max-over-ranks timing) with
two gloo ranks on the CPU: no GPU, no NCCL."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, ms_local, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    try:
        dist.barrier()
        ms_step, value = bench.replica_throughput(ms_local[rank], 4, 1000, world)
        out[rank] = (ms_step, value, bench.max_over_ranks(rank + 0.5, world))
    finally:
        dist.destroy_process_group()


def test_replica_throughput_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    world, port = 2, _free_port()
    ms_local = [40.0, 50.0]            # total ms over 4 steps, per rank
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank, args=(world, port, ms_local, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    for r in range(world):
        ms_step, value, mx = res[r]
        assert ms_step == pytest.approx(50.0 / 4)          # the slowest replica
        assert value == pytest.approx(2 * 1000 / (12.5e-3))  # both replicas' tokens
        assert mx == 1.5


def test_replica_throughput_single_rank():
    import bench
    assert bench.replica_throughput(30.0, 3, 600, 1) == (10.0, 60000.0)
    assert bench.max_over_ranks(7.0, 1) == 7.0
