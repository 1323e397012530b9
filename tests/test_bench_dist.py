"""Host logic of the multi-GPU bench path, on CPU: two gloo ranks check that
the step time is the max over ranks and the job throughput counts every
replica's audio (the bench runs one independent decoder replica per GPU)."""
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


def _rank(rank, world, port, times, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = bench.max_over_ranks(times[rank], world, torch.device("cpu"))
        out[rank] = m
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    times = [120.5, 97.25]
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, times, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0] == pytest.approx(120.5) and out[1] == pytest.approx(120.5)


def test_single_rank_and_throughput():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, None) == 3.5
    # 2 replicas, 10 s of audio each per 40 ms step -> 500 audio-s/s for the job
    assert bench.job_throughput(2, 10.0, 40.0) == pytest.approx(500.0)
    assert bench.job_throughput(1, 10.0, 40.0) == pytest.approx(250.0)
