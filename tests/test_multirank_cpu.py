"""The multi-GPU bench path on CPU: world_size 2 over gloo (127.0.0.1).

With N GPUs every rank runs its own replica (tokens are independent, so there is
no collective on the data path); the only cross-rank steps are the barrier and
the max of the per-rank times. These tests check that host logic: every rank
gets the slowest rank's time, and the job's tokens/s counts all ranks' tokens
over that time.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        ms = bench.max_over_ranks(times[rank], world)
        out[rank] = (ms, bench.job_tokens_per_s(32768, world, 10, ms))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("times", [(100.0, 125.0), (130.0, 90.0)])
def test_max_over_ranks_and_job_rate(times):
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, times, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    slow = max(times)
    for r in range(world):
        ms, rate = out[r]
        assert ms == slow
        assert rate == pytest.approx(32768 * 2 * 10 / (slow / 1e3))


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert bench.job_tokens_per_s(1000, 1, 4, 2000.0) == pytest.approx(2000.0)
