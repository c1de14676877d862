"""The multi-GPU path of the benchmark runs independent replicas (one GPU
holds a layer; no collective is on the data path): each rank times its own
step and the job reports the units of all ranks over the slowest rank's
time.  Checked here with two gloo ranks on the CPU."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    ms_local = [2.0, 3.5][rank]
    ms = bench.replica_max_ms(ms_local, dist)
    rate = bench.replica_rate(1000.0, ms, world)
    q.put((rank, ms, rate))
    dist.barrier()
    dist.destroy_process_group()


def test_replica_max_and_rate_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, rate in out:
        assert ms == 3.5                       # the slowest rank sets the time
        assert rate == pytest.approx(2 * 1000.0 / 3.5e-3)


def test_single_process_passthrough():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.replica_max_ms(1.25) == 1.25
    assert bench.replica_rate(10.0, 2.0, 1) == pytest.approx(5000.0)
