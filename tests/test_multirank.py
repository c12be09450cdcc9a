"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2): each rank
runs an independent replica, the job time is the max over ranks and the
value is the units of all ranks over that time. No data-path collective."""
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
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    ms_local = [12.5, 20.0][rank]
    m = bench.reduce_max(ms_local, dist)
    out[rank] = (m, bench.job_throughput(4096, world, m))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0] == out[1]
    m, v = out[0]
    assert m == 20.0
    assert v == pytest.approx(2 * 4096 / 0.020)


def test_single_rank_identity():
    import bench
    assert bench.reduce_max(3.0) == 3.0
    assert bench.job_throughput(100, 1, 1000.0) == pytest.approx(100.0)
