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


def test_tensor_peak_follows_the_clocks():
    """The 3xTF32 roofline denominator: the burst figure at the maximum clock
    without capping, the sustained figure scaled by the sampled clock under
    capping or a lower clock, and never more than the burst figure."""
    sys.path.insert(0, ROOT)
    import bench
    pk = {"bf16": 1590.0, "bf16_sustained": 1400.0, "sustained_mhz": 1300.0,
          "sm_max_mhz": 1965.0, "source": "fallback"}
    burst = 1590.0 * bench.TF32_PER_BF16 / 3.0
    peak, _, b = bench.tensor_peak(pk, None)
    assert peak == pytest.approx(burst) and b == pytest.approx(burst)
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.tensor_peak(pk, full)[0] == pytest.approx(burst)
    capped_low = {"sm_mhz": 1300.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.tensor_peak(pk, capped_low)[0] == pytest.approx(
        1400.0 * bench.TF32_PER_BF16 / 3.0)
    # a brief cap at the maximum clock: the scaled sustained figure would
    # exceed the burst one, so the burst one is taken
    capped_full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.tensor_peak(pk, capped_full)[0] == pytest.approx(burst)
    slow = {"sm_mhz": 1000.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.tensor_peak(pk, slow)[0] == pytest.approx(
        1400.0 * 1000.0 / 1300.0 * bench.TF32_PER_BF16 / 3.0)


def test_tensor_peak_of_the_fp16_split():
    """The fp16 split conv class takes the bf16 figure at the fp16 rate (1:1
    with bf16) over its three products, under the same clock rules."""
    sys.path.insert(0, ROOT)
    import bench
    pk = {"bf16": 1590.0, "bf16_sustained": 1400.0, "sustained_mhz": 1300.0,
          "sm_max_mhz": 1965.0, "source": "fallback"}
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    peak, src, burst = bench.tensor_peak(pk, full, f16=True)
    assert peak == pytest.approx(530.0) and burst == pytest.approx(530.0)
    assert "3xF16" in src
    capped_low = {"sm_mhz": 1300.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.tensor_peak(pk, capped_low, f16=True)[0] == pytest.approx(1400.0 / 3.0)
    kd = {"avg_launch_ms": 1.0, "flops": 300e9, "bytes": 1e9}
    r = bench.roofline_for("conv1d_tm_f16", kd, pk, full)
    assert r["bound"] == "tensor" and r["frac"] == pytest.approx(300.0 / 530.0)
    r = bench.roofline_for("conv1d_tm", kd, pk, full)
    assert r["frac"] == pytest.approx(300.0 / (1590.0 * bench.TF32_PER_BF16 / 3.0))
