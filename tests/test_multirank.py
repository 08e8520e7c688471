"""The multi-rank path of bench.py on CPU with gloo, world size 2: ranks agree on
the slowest rank's time, the job throughput counts every rank's batch, and the
reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = 10.0 * rank + 5.0               # rank 1 is the slower one
        slowest = bench.reduce_max(local, world)
        out[rank] = (slowest, bench.job_tokens_per_s(world, 64, slowest))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_slowest_time_and_job_throughput():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0][0] == out[1][0] == 15.0
    assert out[0][1] == pytest.approx(2 * 64 / 0.015)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.job_tokens_per_s(1, 64, 8.0) == pytest.approx(8000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")

    class A:
        workload, steps, warmup, cpu_seconds, gpus = "c3", 1, 0, 1.0, 2
    assert bench.run_reference(A()) == 0
    assert capsys.readouterr().out == ""
