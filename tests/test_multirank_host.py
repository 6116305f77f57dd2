"""The multi-rank host logic of bench.py on CPU: two gloo ranks take the same
collective step, agree on the slowest rank's time, and report the whole-job rate
over all ranks' units.  The reference arm does no work on ranks other than 0."""
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


def _rank(rank, world, port, times, out):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(times[rank], world, "cpu")
        v = bench.job_throughput(1.0e9, world, 10, t, "flop")
        ref = bench.run_reference(None, None, None) if rank != 0 else "skipped"
        out.put((rank, t, v, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time_and_the_job_rate():
    world, port = 2, _free_port()
    times = [3.0, 5.0]   # ms for 10 steps on each rank
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, times, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(out.get(timeout=10) for _ in range(world))
    for rank, t, v, ref in got:
        assert t == max(times)
        # 1 GFLOP per step, 2 ranks, 10 steps in 5 ms (the slowest rank): 4 TFLOP/s for the job
        assert v == pytest.approx(1.0e9 * world * 10 / 5e-3 / 1e12)
        if rank != 0:
            assert ref is None        # the oracle arm returns at once on other ranks


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(2.5, 1, "cpu") == 2.5
    assert bench.job_throughput(2.0e9, 1, 4, 8.0, "bytes") == pytest.approx(2.0e9 * 4 / 8e-3 / 1e9)
