"""The multi-GPU path on CPU: world_size-2 gloo ranks.

The method shards by sequence with no exchange: every rank runs its own replica and
only the timing is reduced (maximum over ranks).  These tests run that host-side logic
of bench.py as two gloo processes on 127.0.0.1.
"""

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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench

    local = [0.25, 0.5][rank]  # rank 1 is the slower replica
    value, slowest = bench.job_throughput(units_per_rank_step=4, steps=10, local_seconds=local, world=world,
                                          dist_on=True)
    m = bench.max_over_ranks(float(rank + 1), True)
    dist.barrier()
    out[rank] = (value, slowest, m)
    dist.destroy_process_group()


def test_replicas_report_the_slowest_rank_and_the_whole_job():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        value, slowest, m = res[rank]
        assert slowest == 0.5 and m == 2.0
        assert value == pytest.approx(world * 4 * 10 / 0.5)


def test_single_process_is_identity():
    import bench

    value, slowest = bench.job_throughput(4, 10, 0.5, world=1, dist_on=False)
    assert slowest == 0.5 and value == pytest.approx(80.0)
