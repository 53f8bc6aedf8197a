"""The multi-rank bookkeeping of bench.py, run as two gloo ranks on the CPU: the job's time is
the slowest rank's, its work the sum of every rank's own problem, and every rank takes the same
collective steps."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        ms = [4.0, 7.5][rank]           # per-rank step times
        units = [1.0e12, 3.0e12][rank]  # per-rank work (each rank its own problem)
        slowest = bench.max_over_ranks(ms, world, device="cpu")
        total = bench.sum_over_ranks(units, world, device="cpu")
        rate = bench.job_rate(units, ms, world, device="cpu")
        bench.barrier(world)
        results[rank] = (slowest, total, rate)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_job_time_and_work():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, results))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        got = dict(results)
    assert set(got) == {0, 1}
    for r in range(world):
        slowest, total, rate = got[r]
        assert slowest == 7.5
        assert total == 4.0e12
        assert rate == pytest.approx(4.0e12 / 7.5e-3)
