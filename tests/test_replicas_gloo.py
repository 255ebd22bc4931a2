"""The multi-GPU path of bench.py on CPU: two ranks over the gloo backend.

The decode path does not shard into a collective (every GPU runs an
independent replica), so what the N > 1 launch adds is host logic: the
barrier around the timed region, the maximum of the ranks' device times, the
whole-job throughput computed from it, and the reference arm running on rank
0 only.  These tests run that logic in two processes without a GPU.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms = 10.0 + 5.0 * rank                     # rank 1 is the slower one
        ms_max = bench.max_over_ranks(ms, world)
        gbs = bench.job_gbs(world, 1_000_000, 4, ms_max)
        bench.barrier(world)
        out[rank] = (ms_max, gbs)
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_sum_the_work():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    for rank in range(world):
        ms_max, gbs = out[rank]
        assert ms_max == 15.0                       # the maximum over ranks, seen by every rank
        assert gbs == pytest.approx(2 * 1_000_000 * 4 / 15e-3 / 1e9)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    calls = []
    monkeypatch.setattr(bench, "oracle_sample", lambda frac: calls.append(frac) or [])

    class A:
        ref_frac, warmup, steps = 0.1, 0, 0
    bench.run_reference(A(), 2, 1)                  # rank 1 of 2: returns without work
    assert calls == []
