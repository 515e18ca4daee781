"""The N > 1 path of bench.py on CPU: two gloo ranks through the same set-up, barrier,
max-over-ranks reduction and whole-job rate as a torchrun launch (replicas only: there
is no data-path collective to test)."""

import os
import socket
import types

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    args = types.SimpleNamespace(impl="reference")
    w, r, local = bench.dist_setup(args)
    import torch.distributed as dist
    try:
        bench.barrier(w)
        slowest = bench.allreduce_max(1.0 + rank, w)          # rank r took 1 + r ms
        out[rank] = (w, r, local, dist.get_backend(), slowest,
                     bench.job_rate(w, 10, 1e9, slowest))
        bench.barrier(w)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_sum_the_work():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert sorted(out.keys()) == [0, 1]
    for rank in (0, 1):
        w, r, local, backend, slowest, rate = out[rank]
        assert (w, r, local, backend) == (2, rank, rank, "gloo")
        assert slowest == 2.0
        assert rate == pytest.approx(2 * 10 * 1e9 / 2e-3)


def test_single_rank_needs_no_process_group():
    assert bench.allreduce_max(3.5, 1) == 3.5
    bench.barrier(1)
    assert bench.job_rate(1, 4, 100.0, 2.0) == pytest.approx(4 * 100 / 2e-3)


def test_reference_arm_runs_on_rank_zero_only():
    args = types.SimpleNamespace(steps=1, warmup=0, impl="reference")
    assert bench.run_reference(args, world=2, rank=1) is None
