"""The N > 1 bench path on CPU: two gloo ranks exercise the barrier, the
max-over-ranks timing reduction and the whole-job throughput that
``bench.py --gpus N`` uses (each GPU runs an independent replica)."""
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


def _rank_main(rank, world, port, results):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms = [4.0, 5.5][rank]  # rank 1 is the slower one
        ms_max = bench.max_over_ranks(ms, world)
        value = bench.job_throughput(world, 1000.0, ms_max)
        bench.barrier(world)
        results[rank] = (ms_max, value)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_by_the_slowest():
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(2):
        ms_max, value = results[r]
        assert ms_max == 5.5
        assert value == pytest.approx(2 * 1000.0 / 5.5e-3)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.job_throughput(1, 10.0, 2.0) == pytest.approx(5000.0)
