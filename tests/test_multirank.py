"""The N > 1 host path of bench.py on CPU: world_size-2 gloo ranks (no GPU).

bench.py runs one replica per GPU (weak scaling; the batch rows are independent, so there is no
collective on the data path).  What crosses ranks is the timing: each rank's step time, reduced to
the maximum over ranks, and the whole-job value computed from it.  These tests run that logic on two
gloo ranks.
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


def _rank_main(rank, world, port, step_ms, out_q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms_max = bench.max_over_ranks(step_ms[rank], "cpu", world)
        value = bench.job_value(world, ms_max)
        out_q.put((rank, ms_max, value))
    finally:
        dist.destroy_process_group()


def _run(world, step_ms):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, step_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    return sorted(q.get(timeout=5) for _ in range(world))


def test_two_ranks_agree_on_the_slowest_step():
    res = _run(2, [0.150, 0.162])
    for rank, ms_max, value in res:
        assert ms_max == pytest.approx(0.162)
        assert value == pytest.approx(2 * 32 / 0.162e-3)   # 2 ranks x 32 queries per slowest step


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.5, "cpu", 1) == 0.5
    assert bench.job_value(1, 0.25) == pytest.approx(32 / 0.25e-3)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        steps, warmup = 3, 3

    bench.run_reference(Args(), 1, 2)   # a non-zero rank returns at once, printing nothing
    assert capsys.readouterr().out == ""
