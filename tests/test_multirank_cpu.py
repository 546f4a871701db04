"""The multi-GPU host logic of bench.py on CPU: two gloo ranks, as torchrun
would launch two GPU ranks.  Every rank runs its own replica (weak scaling);
the job time is the slowest rank's and the job throughput counts all ranks."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [120.0, 150.0][rank]
        m = bench.max_over_ranks(local_ms)
        w, r, lr = bench.dist_env()
        value = bench.job_throughput(2.0 * 2048 * 5120 * 20480, 100, w, m)
        out[rank] = (m, w, r, lr, value)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_weak_scaling_throughput():
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 150.0              # slowest rank's time on both
    assert [res[i][1:4] for i in (0, 1)] == [(2, 0, 0), (2, 1, 1)]
    ops = 2.0 * 2048 * 5120 * 20480
    assert res[0][4] == pytest.approx(ops * 100 * 2 / 0.150 / 1e12)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(1e12, 10, 1, 1000.0) == pytest.approx(10.0)
