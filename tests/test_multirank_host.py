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


# ------------------------------------------------------------------ context-parallel ring (host logic)

def _cp_rank(rank, world, port, out):
    """One gloo rank of the ring forward.  The per-chunk attention and the merge are
    the fp64 oracle's (no GPU here); what runs for real is the schedule and the
    point-to-point exchange of the K/V chunks around the ring."""
    sys.path.insert(0, ROOT)
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    import workloads as W
    from exact_attention_131_b200 import cp

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        L = 17
        c = W.dense_case(1, 4, 2, world * L, world * L, 16, dtype="f32", causal=True, sinks=True, seed=60)
        sl = slice(rank * L, (rank + 1) * L)
        q, k, v = (torch.from_numpy(np.ascontiguousarray(x[:, :, sl])) for x in (c.q, c.k, c.v))
        seen = []

        def attn(q_, k_, v_, *, causal, scale):
            seen.append(bool(causal))
            o, lse = oracle.attn(q_.numpy(), k_.numpy(), v_.numpy(), scale=scale, causal=causal)
            return torch.from_numpy(o), torch.from_numpy(lse)

        def merge(o_parts, lse_parts, *, sinks, sink_rows):
            rows = np.broadcast_to(np.asarray(sinks, np.float64)[None, :, None], lse_parts[0].shape)
            o, lse = oracle.merge([x.numpy() for x in o_parts], [x.numpy() for x in lse_parts], sink_rows=rows)
            return torch.from_numpy(o), torch.from_numpy(lse)

        o, lse = cp.ring_attention_forward(q, k, v, causal=True, scale=c.scale, sinks=c.sinks, attn=attn, merge=merge)
        ro, rl = oracle.attn(c.q, c.k, c.v, scale=c.scale, causal=True, sinks=c.sinks)
        out.put((rank, float(np.abs(o.numpy() - ro[:, :, sl]).max()), float(np.abs(lse.numpy() - rl[:, :, sl]).max()),
                 seen))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ring_forward_over_gloo_ranks_equals_attention_over_the_whole_sequence(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_cp_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    got = sorted(out.get(timeout=10) for _ in range(world))
    for rank, d_o, d_l, seen in got:
        assert d_o < 1e-10 and d_l < 1e-10, (rank, d_o, d_l)
        # rank r attends to its own chunk under the mask first, then to the r earlier chunks unmasked
        assert seen == [True] + [False] * rank


def test_ring_schedule():
    sys.path.insert(0, ROOT)
    from exact_attention_131_b200 import cp

    assert cp.ring_schedule(2, 4, True) == [(0, 2, True), (1, 1, False), (2, 0, False), (3, 3, None)]
    assert cp.ring_schedule(0, 3, True) == [(0, 0, True), (1, 2, None), (2, 1, None)]
    assert [m for _, _, m in cp.ring_schedule(1, 3, False)] == [False] * 3
    for world in range(1, 6):
        for rank in range(world):
            srcs = [s for _, s, _ in cp.ring_schedule(rank, world, True)]
            assert sorted(srcs) == list(range(world))          # every chunk passes by once
