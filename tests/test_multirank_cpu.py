"""The N > 1 host path of bench.py on CPU: two gloo ranks (world size 2).

On GPUs every rank runs its own copy of the workload (weak scaling; the
attention path has no cross-rank exchange), the timed interval is the max over
ranks and the reported value is the work of all ranks over that interval.
These tests run the same helpers over a gloo process group on the host.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, per_rank_ms, out):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        dist.barrier()
        ms_max = bench.rank_max(per_rank_ms[rank], world)
        e2e_max = bench.rank_max(10.0 * per_rank_ms[rank], world)
        dist.barrier()
        out[rank] = (ms_max, e2e_max, bench.rank_seed(rank))
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_ranks():
    per_rank_ms = [3.5, 7.25]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(2, _free_port(), per_rank_ms, out), nprocs=2, join=True,
                           start_method="spawn")
        return per_rank_ms, dict(out)


def test_every_rank_sees_the_slowest_rank(two_ranks):
    per_rank_ms, out = two_ranks
    assert sorted(out) == [0, 1]
    for r in (0, 1):
        assert out[r][0] == max(per_rank_ms)
        assert out[r][1] == 10.0 * max(per_rank_ms)


def test_rank_copies_have_distinct_seeds_and_equal_shapes(two_ranks):
    _, out = two_ranks
    s0, s1 = out[0][2], out[1][2]
    assert s0 != s1
    w0 = workloads.make("tiny", seed=s0)
    w1 = workloads.make("tiny", seed=s1)
    assert w0.q.shape == w1.q.shape and w0.flops_total() == w1.flops_total()
    assert not (w0.q == w1.q).all()


def test_aggregate_is_all_ranks_work_over_the_slowest_time():
    # 2 ranks, 45.097 GFLOP per rank-step, 100 steps, slowest rank 12.8 ms
    v = bench.aggregate_tflops(2, 45.097e9, 100, 12.8)
    assert v == pytest.approx(2 * 45.097e9 * 100 / 12.8e-3 / 1e12)
    # weak scaling: per-rank work fixed, so two ranks at the same speed double the value
    assert bench.aggregate_tflops(2, 1e12, 1, 1000.0) == pytest.approx(2 * bench.aggregate_tflops(1, 1e12, 1, 1000.0))


def test_single_rank_max_is_identity():
    assert bench.rank_max(4.5, 1) == 4.5


def test_reference_arm_other_ranks_exit_without_work(capsys):
    class A:
        steps, warmup, mode, beta = 1, 0, 1, 2.0

    assert bench.run_reference(A(), rank=1, world=2) == 0
    assert capsys.readouterr().out == ""
