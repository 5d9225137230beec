"""Multi-process host logic on CPU (gloo, world size 2): the bench's job time is the max over
ranks; every rank runs its own replica (no data-path collective on this path)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    per_rank = [[0.110, 0.250, 0.130], [0.125, 0.240, 0.150]][rank]   # ms: hsa, dense, e2e
    got = bench.max_over_ranks(per_rank, dist, torch.device("cpu"))
    out[rank] = got
    dist.barrier()
    dist.destroy_process_group()


def test_timing_is_max_over_two_gloo_ranks():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
        res = dict(out)
    for r in (0, 1):
        assert res[r] == pytest.approx([0.125, 0.250, 0.150])


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks([1.0, 2.0], None, torch.device("cpu")) == [1.0, 2.0]
