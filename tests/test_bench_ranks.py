"""bench.py's multi-rank logic on CPU: two `gloo` ranks on 127.0.0.1.

Under torchrun every rank runs its own replica of the workload (weak
scaling, no data-path collective); the only cross-rank steps are barriers
and the max over ranks of each timed region.  These tests run that logic
with CPU process groups, no GPU needed.
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


def _rank_main(rank, world, port, elapsed, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        mx = bench.max_over_ranks(elapsed[rank], world)
        bench.barrier(world)
        q.put((rank, mx, bench.job_us_per_call(mx, 10, world)))
    finally:
        dist.destroy_process_group()


def _run_ranks(elapsed):
    world = len(elapsed)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, elapsed, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, mx, us = q.get(timeout=120)
        got[rank] = (mx, us)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return got


def test_max_over_ranks_takes_the_slowest_rank():
    # rank 1 is the slow one: both ranks must report its time
    got = _run_ranks([1.25, 3.5])
    assert got[0][0] == got[1][0] == 3.5
    # 2 ranks x 10 calls in 3.5 ms: 175 us per call for the whole job
    assert got[0][1] == pytest.approx(175.0)


def test_max_over_ranks_is_order_independent():
    got = _run_ranks([9.0, 2.0])
    assert got[0][0] == got[1][0] == 9.0


def test_single_rank_needs_no_process_group():
    assert not dist.is_initialized()
    assert bench.max_over_ranks(4.0, 1) == 4.0
    bench.barrier(1)   # a no-op without torchrun
    assert bench.job_us_per_call(4.0, 20, 1) == pytest.approx(200.0)


def test_weak_scaling_value_counts_every_rank_calls():
    # the same per-rank time on 1, 2, 4, 8 ranks: the job does N times the
    # calls, so the whole-job time per call falls as 1/N
    vals = [bench.job_us_per_call(13.0, 200, n) for n in (1, 2, 4, 8)]
    assert vals[0] == pytest.approx(65.0)
    for n, v in zip((1, 2, 4, 8), vals):
        assert v * n == pytest.approx(vals[0])


def test_reference_arm_prints_only_on_rank_zero(capsys):
    class Args:
        workload = "tiny"
        warmup = 3
        steps = 1
        ref_rows = 2
        gpus = 2
    bench.run_reference(Args(), world=2, rank=1)
    assert capsys.readouterr().out == ""
