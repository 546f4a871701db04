"""The column-parallel (N-split) host logic on CPU: the column slices, and
two gloo ranks assembling Y from their column slices.  Each rank's slice is
computed by the oracle, standing in for the rank's GPU forward (the kernels
themselves are covered by the GPU parity tests, including sharded weights):
what is checked here is that slicing W by columns and gathering reproduces
the unsharded result exactly."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from int8_quantized_matmul_outlier_b200.nsplit import column_ranges, gather_columns


def test_column_ranges_cover_align_and_balance():
    for N, world in [(16, 1), (784, 2), (784, 3), (20480, 8), (49152, 8), (48, 3), (80, 2)]:
        r = column_ranges(N, world)
        assert len(r) == world and r[0][0] == 0 and r[-1][1] == N
        assert all(a1 == b0 for (_, a1), (b0, _) in zip(r, r[1:]))
        widths = [b - a for a, b in r]
        assert all(w % 16 == 0 and w >= 16 for w in widths)
        assert max(widths) - min(widths) <= 16
    for N, world in [(32, 3), (40, 1), (0, 1)]:
        with pytest.raises(ValueError):
            column_ranges(N, world)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import oracle
    import workloads
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        res = {}
        for M, K, N, n_out in ((24, 64, 80, 2), (7, 256, 96, 3)):
            p = workloads.small(M, K, N, n_out, seed=M + K + N)
            ranges = column_ranges(N, world)
            a, b = ranges[rank]
            part = oracle.decomp_matmul(p.X, np.ascontiguousarray(p.W[:, a:b]), p.alpha)["Y"]
            Y = gather_columns(torch.from_numpy(np.ascontiguousarray(part)), ranges)
            full = oracle.decomp_matmul(p.X, p.W, p.alpha)["Y"]
            same_bits = (Y.view(torch.int16).numpy() == full.view(np.int16)).all()
            res[(M, N)] = bool(same_bits) and tuple(Y.shape) == (M, N)
        try:
            gather_columns(torch.zeros((4, 16), dtype=torch.float16), column_ranges(64, world))
            res["shape_check"] = False
        except ValueError:
            res["shape_check"] = True
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_two_ranks_gather_column_slices_into_the_unsharded_result():
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for r in (0, 1):
        assert all(res[r].values()), res[r]


def test_single_process_gather_is_identity():
    Y = torch.arange(32, dtype=torch.float16).reshape(2, 16)
    assert gather_columns(Y, [(0, 16)]) is Y
