"""The benchmark's multi-rank host logic on two CPU ranks over gloo.

bench.py runs one independent replica of the call per GPU (weak scaling);
the only cross-rank steps are barriers and the max-over-ranks reduction of
the timings, checked here without a GPU.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        step_ms = [12.5, 20.0][rank]
        mx = bench.reduce_max(step_ms, world)
        dist.barrier()
        q.put((rank, mx, bench.whole_job_ms_per_call(mx, 1, world)))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_whole_job_rate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [20.0, 20.0]          # every rank sees the slowest rank's time
    assert [r[2] for r in res] == [10.0, 10.0]          # two calls complete per 20 ms step


def test_single_rank_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.whole_job_ms_per_call(8.0, 1, 1) == 8.0
    assert bench.executed_fine_flops(1, 40, 39936, 32, 128) == pytest.approx(1.675e12, rel=1e-3)
    assert bench.executed_fine_flops(1, 40, 39936, 624, 128) == pytest.approx(32.66e12, rel=1e-3)
