"""Multi-GPU host logic of the benchmark on CPU: world size 2 over gloo.

bench.py runs one independent replica per rank (no collective on the data path);
the only cross-rank steps are the barriers around the timed region and the
max-over-ranks of the measured time.  Both run here over gloo with two processes.
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world, rank)
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, torch.device("cpu"))
        val = bench.job_value(world, 32768, ms)
        bench.barrier(world, rank)
        q.put((rank, ms, val))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_takes_the_slowest_rank():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms, val in res:
        assert ms == 15.0                                  # max over ranks
        assert val == pytest.approx(2 * 32768 / 0.015)     # all ranks' tokens / slowest time


def test_job_value_single_rank():
    import bench
    assert bench.job_value(1, 32768, 80.0) == pytest.approx(32768 / 0.08)
