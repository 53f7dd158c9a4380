"""The multi-GPU bench logic, run as two gloo ranks on the CPU.

Each rank decodes its own sequences (its own seed namespace); the only
cross-rank traffic is the barrier and the max-over-ranks reduction of the
timed region, from which rank 0 reports whole-job throughput.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        ms = 100.0 + 50.0 * rank  # rank 1 is the slow one
        m = bench.max_over_ranks(ms, "cpu")
        out[rank] = (m, bench.job_value(1000, 4, world, m), bench.rank_tag("w", rank))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 150.0
    assert res[0][1] == pytest.approx(2 * 1000 * 4 / 0.150)
    assert res[0][2] != res[1][2]  # ranks draw distinct sequences


def test_single_process_is_identity():
    assert bench.max_over_ranks(12.5, "cpu") == 12.5
    assert bench.job_value(10, 3, 1, 1000.0) == pytest.approx(30.0)
