"""The N > 1 path of the benchmark on CPU: two gloo ranks (independent replicas, no data-path
collective) agree on the max-over-ranks timing, and the whole-job rate counts every rank's units."""
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


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [4.0 + rank, 9.0 - rank, 0.25 * (rank + 1)]       # this rank's step, e2e, kernel times
        got = bench.max_over_ranks(ms, "cpu")
        dist.barrier()
        out[rank] = got + [bench.whole_job_rate(1.0e9, world, got[0])]
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_max_and_whole_job_rate():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    assert out[0] == out[1]
    step, e2e, kern, rate = out[0]
    assert (step, e2e, kern) == (5.0, 9.0, 0.5)
    assert rate == pytest.approx(2 * 1.0e9 / 5.0e-3)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks([1.5, 2.5], "cpu") == [1.5, 2.5]
    assert bench.whole_job_rate(100.0, 1, 1000.0) == pytest.approx(100.0)
