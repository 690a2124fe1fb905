"""The multi-rank bench path on the CPU: two gloo ranks over 127.0.0.1.

Sequences are independent, so the bench shares no data between ranks; the only
cross-rank step is the max of the timed duration, taken after the timed region.
These tests run that step and the throughput formula on two real processes,
and check that the reference arm runs on rank 0 alone."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms_local = [12.5, 30.25][rank]  # the ranks' own timed durations
        ms_max = bench.max_over_ranks(ms_local, dist, torch.device("cpu"))
        out.put((rank, ms_max, bench.job_throughput(world, 32, 100, ms_max)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[1] for g in got] == [30.25, 30.25], "every rank must see the slowest rank's time"
    # 2 ranks x 32 sequences x 100 steps over 30.25 ms
    assert got[0][2] == pytest.approx(2 * 32 * 100 / 0.03025)
    assert got[0][2] == got[1][2]


def test_single_process_is_identity():
    assert bench.max_over_ranks(7.0, None, None) == 7.0
    assert bench.job_throughput(1, 32, 10, 2.0) == pytest.approx(160000.0)


def test_reference_arm_runs_on_rank_zero_only():
    class Args:
        warmup, steps = 3, 2
    assert bench.run_reference(Args(), rank=1, world=2) is None
