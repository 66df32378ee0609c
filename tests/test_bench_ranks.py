"""Host logic of the multi-GPU bench path on CPU: two gloo ranks.

Every rank runs its own replica of the workload; the timed region is the max
over ranks and the job's throughput counts every rank's FLOPs. No GPU."""

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


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        results[rank] = bench.max_over_ranks(local_ms)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    results = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), results), nprocs=world, join=True)
    assert results[0] == results[1] == 15.0


def test_max_over_ranks_without_a_group_is_identity():
    assert not dist.is_initialized()
    assert bench.max_over_ranks(3.5) == 3.5


def test_aggregate_counts_every_replica():
    ms_per_step, tflops = bench.aggregate(step_flops=2e12, world=4, ms_total_max=40.0, steps=10)
    assert ms_per_step == pytest.approx(4.0)
    assert tflops == pytest.approx(4 * 2e12 / 4e-3 / 1e12)


def test_reference_arm_non_zero_rank_exits_without_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")

    class A:
        steps, warmup, gpus = 1, 1, 2

    assert bench.run_reference(A()) == 0
    assert capsys.readouterr().out == ""
