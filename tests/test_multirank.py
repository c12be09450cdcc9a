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


def test_reference_arm_under_torchrun_prints_one_line():
    """bench.py --impl reference launched under torchrun for N > 1
    (torchrun, two ranks): rank 0 alone runs the oracle and prints the one
    JSON line; the other rank exits 0 without work."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "2", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    for k in ("metric", "unit", "higher_is_better", "config", "cpu_baseline", "e2e"):
        assert k in d
