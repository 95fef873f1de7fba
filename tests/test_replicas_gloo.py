"""The multi-GPU benchmark path runs independent replicas (no data-path
collective): its only cross-rank steps are the barrier and the max-over-ranks
timing.  Exercised here with two gloo ranks on the CPU."""

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


def _rank_main(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        ms = bench.max_over_ranks(torch, dist, times[rank], torch.device("cpu"))
        out[rank] = (ms, bench.job_rate(world, 1000, 10, ms))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_job_rate(world):
    times = [3.0, 5.0]
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), times, out), nprocs=world, join=True)
    for r in range(world):
        ms, rate = out[r]
        assert ms == 5.0                           # every rank reports the slowest time
        assert rate == pytest.approx(world * 1000 * 10 / 5e-3 / 1e9)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(torch, None, 4.5, torch.device("cpu")) == 4.5
    assert bench.job_rate(1, 2e9, 1, 1000.0) == pytest.approx(2.0)


def test_reference_arm_other_ranks_do_nothing(capsys):
    class A:
        steps, warmup = 1, 0

    bench.run_reference(A(), rank=1, world=2)
    assert capsys.readouterr().out == ""
