"""The multi-rank path of bench.py on CPU: two gloo ranks (world size 2),
no GPU.  The sweep does not shard (replicas only), so the only exchange is
the timing reduction: every rank must see the slowest rank's time, and the
whole-job value counts every rank's work against that time."""
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


def _rank_main(rank, world, port, step_ms, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(step_ms[rank], True, "cpu")
        dist.barrier()
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_every_rank_sees_the_slowest_rank_time():
    world = 2
    step_ms = [1.25, 3.5]
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), step_ms, out), nprocs=world, join=True)
        assert dict(out) == {0: 3.5, 1: 3.5}


def test_single_rank_and_whole_job_value():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, False, "cpu") == 2.5
    # two ranks, each 1 TFLOP of work per step, slowest step 2 ms: 1000 TFLOP/s
    assert bench.whole_job_tflops(2, 1e12, 2.0) == pytest.approx(1000.0)
    assert bench.whole_job_tflops(1, 1e12, 2.0) == pytest.approx(500.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import bench
    # a rank other than 0 returns at once (before reading its arguments),
    # prints nothing and does no work
    bench.reference_arm(None, 1)
    assert capsys.readouterr().out == ""
