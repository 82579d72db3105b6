"""Multi-process host logic of the benchmark on CPU (gloo, world size 2):
timings are reduced as the max over ranks, the job value is amortised over
ranks and steps, and the reference arm runs on rank 0 only."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
    m = bench.max_over_ranks(local_ms, torch.device("cpu"))
    out[rank] = m
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert out[0] == 15.0 and out[1] == 15.0


def test_job_value_amortised():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks, 10 steps, slowest rank 200 ms in total: 20 layers in 200 ms
    assert bench.job_ms_per_layer(200.0, 10, 2) == 10.0
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5   # not distributed: identity


def test_reference_arm_only_on_rank0(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")

    class A:
        workload = "tiny"
        warmup = 1
        steps = 1
        cpu_seconds = 0.1
        gpus = 2

    bench.run_reference(A)
    assert capsys.readouterr().out == ""
