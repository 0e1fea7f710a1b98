"""The multi-rank path of bench.py on CPU: two ranks on the gloo backend.

With N GPUs the bench runs one independent replica of the layer per rank (the path does
not shard), so the only cross-rank steps are the barrier and the max-over-ranks reduction
of the timings; the whole-job value is every rank's units over the slowest rank's time.
These tests run exactly those helpers with world_size 2 (gloo, 127.0.0.1), plus the
reference arm's rule that only rank 0 works.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # rank r "measured" these (ms of the timed steps, ms of the e2e steps)
        local = [10.0 + 5.0 * rank, 30.0 - 7.0 * rank]
        dist.barrier()
        got = bench.max_over_ranks(local, world, "cpu")
        out[rank] = got + [bench.job_rate(64, world, got[0])]
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        total, e2e, rate = out[r]
        assert total == 15.0            # the slowest rank's timed interval
        assert e2e == 30.0              # each value reduced on its own
        assert rate == pytest.approx(64 * world / 15.0e-3)


def test_single_rank_reduction_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5], 1) == [1.5, 2.5]
    assert bench.job_rate(10, 1, 2.0) == pytest.approx(5000.0)


def test_reference_arm_works_on_rank_zero_only():
    import bench
    # any rank other than 0 returns before reading its arguments or touching the oracle
    assert bench.run_reference(None, 1) is None
