"""The N > 1 path of bench.py on CPU: two gloo ranks, each timing its own
replica; the step time is the max over ranks and the throughput counts every
rank's tokens.  (The data path has no collective: ranks are replicas.)"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms_local = 10.0 + 5.0 * rank          # rank 1 is the slow one
        ms = bench.reduce_max_ms(ms_local, world)
        value = bench.aggregate_value(tokens_per_rank_step=8192, world=world, steps=4, ms_max=ms)
        out[rank] = (ms, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_timing_and_aggregate():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    assert out[0][0] == pytest.approx(15.0) and out[1][0] == pytest.approx(15.0)
    expect = 8192 * 2 * 4 / 0.015
    assert out[0][1] == pytest.approx(expect) and out[1][1] == pytest.approx(expect)
