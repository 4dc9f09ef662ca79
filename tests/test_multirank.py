"""The N > 1 host logic of bench.py on CPU: two gloo ranks, each timing its own
replica, reduce to the slowest rank's time and the whole job's throughput."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    local_ms = [12.0, 20.0][rank]           # rank 1 is the slow one
    ms, value = bench.job_throughput(local_ms, units_per_rank=640, dist=dist, device="cpu")
    q.put((rank, ms, value))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_throughput_is_max_time_over_all_units():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value in out:
        assert ms == 20.0                                  # max over ranks
        assert value == pytest.approx(2 * 640 / 0.020)     # all ranks' tokens / slowest time


def test_single_rank_throughput():
    import bench
    ms, value = bench.job_throughput(4.0, 100, None, "cpu")
    assert ms == 4.0 and value == pytest.approx(100 / 0.004)
