#!/usr/bin/env python
"""Decoder throughput on B200: seconds of audio decoded per second.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the plain CPU oracle, timed on the host

One step = one whole decode (conv_pre, every ConvT stage with its AMP blocks,
act_post, conv_post, final op) of one batch of the workload, weights and
latent resident in HBM.  With N > 1 (torchrun) every rank decodes its own
batch on its own GPU (independent replicas, no collective on the data path);
the step time is the max over ranks.  Prints one JSON line on rank 0.
"""
import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bigvgan_waveform_decoder_alias_b200 import synth  # noqa: E402

METRIC = "audio-seconds decoded per second (1 B200); activation GB/s and conv pipe % of peak"
UNIT = "audio_s/s"
L2_FLUSH_BYTES = 256 << 20  # twice the 126 MB L2
SMS = 148
FP32_LANES_PER_SM = 128


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=synth.H3_60S_TILED.name,
                    choices=sorted(synth.DECODER_WORKLOADS))
    ap.add_argument("--activation-sweep", action="store_true",
                    help="time the activation over the C x T sweep grid (B = 2) instead of "
                         "the decoder; one JSON line with every shape")
    ap.add_argument("--cpu-sample-frames", type=int, default=40,
                    help="latent frames (one side) of the oracle's timed sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tf32-only", action="store_true",
                    help="decode with every tensor-core conv in 3xTF32 (bv_decoder_config."
                         "tf32_only); by default the AMP and transposed convs that qualify use "
                         "the fp16 split and the line also reports the 3xTF32 decode")
    ap.add_argument("--case", default=None,
                    help="time one kernel on one shape instead of the decoder (for profiling): "
                         "activation:BxCxT | conv1d:BxCxT:K:d | convt:BxCinxT:Cout:s | "
                         "actconv:BxCxT:K:d (activation then conv, the decoder's kernels) | "
                         "amp:BxCxT:K (an AMP block, dilations 1, 3, 5) | "
                         "frontend:CxSxT:Cout (latent de-normalisation + dec_in) | "
                         "dav:FRAMES (the Music-3 DAV decoder on a stereo latent) | "
                         "bwe:FRAMES (the LTX bandwidth-extension tail on FRAMES mel hops of "
                         "stereo 16 kHz input)")
    return ap.parse_args()


def run_case(args):
    """One kernel on one seeded shape, W warm-up and K timed launches."""
    import torch
    from bigvgan_waveform_decoder_alias_b200 import native
    kind, shape, *rest = args.case.split(":")
    s = synth.NormalStream(7)
    filt = torch.from_numpy(native.bv_filter_design()).cuda()
    if kind in ("dav", "bwe"):
        # whole decoders: the unit is audio-seconds of output per second
        frames = int(shape)
        if kind == "dav":
            geo = synth.MUSIC3_DAV
            z = torch.from_numpy(s.normal((2, geo.latent_channels, frames))).cuda()
            dec = native.DavDecoder(geo, synth.draw_dav_params(s, geo))
            y = dec.decode(z)
            ws = torch.empty(native.lib().bv_dav_workspace_size(
                ctypes.byref(dec.cfg), 2, frames) // 4 + 64, device="cuda")
            fn = lambda: dec.decode(z, y=y, workspace=ws)  # noqa: E731
            work = frames * geo.hop / geo.sample_rate
        else:
            geo, sp = synth.LTX_BWE, synth.LTX_BWE_SPEC
            low = torch.from_numpy(0.3 * s.normal((2, frames * sp.hop))).cuda()
            params = synth._draw_params(s, synth.param_layout(geo))
            basis, mel = sp.bases()
            tail = native.BweTail(geo, params, sp, basis, mel, filt=filt.cpu().numpy())
            y = tail(low)
            ws = torch.empty(native.lib().bv_bwe_tail_workspace_size(
                ctypes.byref(tail.dec.cfg), 2, frames * sp.hop, sp.n_fft, sp.hop, sp.n_mels,
                sp.ratio) // 4 + 64, device="cuda")
            fn = lambda: tail(low, y=y, workspace=ws)  # noqa: E731
            work = frames * sp.hop / sp.in_rate
        unit = "audio_s/s"
        return _time_case(args, native, fn, work, unit)
    B, C, T = (int(v) for v in shape.split("x"))
    x = torch.from_numpy(s.normal((B, C, T))).cuda()
    if kind == "frontend":
        # z [C, S, T] with S = B sides here: C latent channels x S x T frames
        Cl, S, Tf, Cout = B, C, T, int(rest[0])
        mean = torch.from_numpy(s.normal((Cl,), 0.0, 0.5)).cuda()
        std = torch.from_numpy(np.abs(s.normal((Cl,), 1.0, 0.3)) + 0.1).cuda()
        w = torch.from_numpy(s.normal((Cout, Cl, 1), 0.0, 0.2)).cuda()
        b = torch.from_numpy(s.normal((Cout,), 0.0, 0.1)).cuda()
        out = torch.empty((S, Cout, Tf), device="cuda")
        fn = lambda: native.bv_latent_front_end(x, mean, std, w, b, out=out)  # noqa: E731
        return _time_case(args, native, fn, 4.0 * (Cl + Cout) * S * Tf, "GB/s")
    if kind == "activation":
        la = torch.from_numpy(s.normal((C,), 0, 0.1)).cuda()
        lb = torch.from_numpy(s.normal((C,), 0, 0.1)).cuda()
        y = torch.empty_like(x)
        fn = lambda: native.bv_activation1d(x, la, lb, filt, y=y)  # noqa: E731
        work, unit = 8.0 * B * C * T, "GB/s"
    elif kind == "conv1d":
        K, d = int(rest[0]), int(rest[1])
        w = torch.from_numpy(s.normal((C, C, K), 0, 0.02)).cuda()
        b = torch.from_numpy(s.normal((C,), 0, 0.02)).cuda()
        y = torch.empty_like(x)
        fn = lambda: native.bv_conv1d(x, w, b, d, (K * d - d) // 2, y=y)  # noqa: E731
        work, unit = 2.0 * B * C * C * K * T, "TFLOP/s"
    elif kind == "convt":
        Co, st = int(rest[0]), int(rest[1])
        w = torch.from_numpy(s.normal((C, Co, 2 * st), 0, 0.02)).cuda()
        b = torch.from_numpy(s.normal((Co,), 0, 0.02)).cuda()
        fn = lambda: native.bv_conv_transpose1d(x, w, b, st)  # noqa: E731
        work, unit = 2.0 * B * C * Co * 2 * st * T, "TFLOP/s"
    elif kind == "actconv":
        # one AMP-block step on the decoder's kernels: activation -> conv
        K, d = int(rest[0]), int(rest[1])
        la = torch.from_numpy(s.normal((C,), 0, 0.1)).cuda()
        lb = torch.from_numpy(s.normal((C,), 0, 0.1)).cuda()
        w = torch.from_numpy(s.normal((C, C, K), 0, 0.02)).cuda()
        b = torch.from_numpy(s.normal((C,), 0, 0.02)).cuda()
        y = torch.empty_like(x)
        ws = torch.empty(native.lib().bv_act_conv1d_workspace_size(B, C, T, C, K, d) // 4 + 64,
                         device="cuda")
        fn = lambda: native.bv_act_conv1d(x, la, lb, filt, w, b, d, y=y, workspace=ws)  # noqa: E731
        work, unit = 2.0 * B * C * C * K * T, "TFLOP/s"
    elif kind == "amp":
        K = int(rest[0])
        wl = synth.AmpWorkload("case", B, C, T, K, (1, 3, 5), seed=7)
        xa, flat = wl.make()
        x = torch.from_numpy(xa).cuda()
        tens, off = {}, 0
        for name, shape, _ in wl.layout():
            n = int(np.prod(shape))
            tens[name] = torch.from_numpy(flat[off:off + n].reshape(shape)).cuda()
            off += n
        p = native.amp_params(K, (1, 3, 5), tens, filt)
        y = torch.empty_like(x)
        ws = torch.empty(native.bv_amp_block_workspace_size_tc(B, C, T, p) // 4 + 64,
                         device="cuda")
        fn = lambda: native.bv_amp_block(x, p, y=y, workspace=ws)  # noqa: E731
        # the block's 6 convs (useful FLOPs); its activations are not counted
        work, unit = 2.0 * 6 * B * C * C * K * T, "TFLOP/s"
    else:
        raise SystemExit(f"unknown case {kind}")
    return _time_case(args, native, fn, work, unit)


def _time_case(args, native, fn, work, unit):
    """W warm-up calls, K calls timed with CUDA events on the current stream
    (median), then a pass with the library's per-class timers."""
    import torch
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for a, b_ in ev:
        a.record()
        fn()
        b_.record()
    torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b_) for a, b_ in ev)
    rate = work / (ms / 1000) / {"GB/s": 1e9, "TFLOP/s": 1e12}.get(unit, 1.0)
    # a second pass with the library's per-class event timers: the mean time
    # of each kernel class per call (for cases that launch several kernels)
    native.timing_reset()
    native.timing(True)
    for _ in range(args.steps):
        fn()
    torch.cuda.synchronize()
    per_class = native.timing_read()
    native.timing(False)
    native.timing_reset()
    classes = {k: {"ms_per_call": v["ms"] / args.steps,
                   "GB/s": v["bytes"] / (v["ms"] / 1000) / 1e9 if v["ms"] > 0 else None,
                   "TFLOP/s": v["flops"] / (v["ms"] / 1000) / 1e12 if v["ms"] > 0 else None}
               for k, v in per_class.items()}
    print(json.dumps({"case": args.case, "ms_median": ms, "achieved": rate, "unit": unit,
                      "steps": args.steps, "warmup": args.warmup, "classes": classes}))
    return 0


# dense TF32 / BF16 tensor throughput, nominal (1.1 vs 2.25 PFLOP/s per B200)
TF32_PER_BF16 = 1.1 / 2.25


def peaks():
    """Roofline denominators: the measured copy bandwidth and bf16 GEMM
    rates of this machine's B200s (a burst, and a seconds-long loop under the
    power cap with the SM clock it settled at), else the profiling recipe's
    fallback (1.59 PFLOP/s burst, about 1.4 sustained near 1.3 GHz)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    out = {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0,
           "sustained_mhz": 1300.0, "sm_max_mhz": 1965.0, "source": "fallback"}
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        out["source"] = "measured"
        out["hbm_gbs"] = float(d.get("hbm_gbs", out["hbm_gbs"]))
        out["bf16"] = float(d.get("bf16_tflops", out["bf16"]))
        out["bf16_sustained"] = float(d.get("bf16_tflops_sustained", out["bf16_sustained"]))
        flat = {}

        def walk(v, pre=""):
            if isinstance(v, dict):
                for k, x in v.items():
                    walk(x, f"{pre}{k}.")
            elif isinstance(v, (int, float)):
                flat[pre[:-1]] = float(v)
        walk(d)
        for k, v in flat.items():  # the clock the sustained figure was measured at
            kl = k.lower()
            if "mhz" in kl and "sustain" in kl and "max" not in kl:
                out["sustained_mhz"] = v
            elif "mhz" in kl and "max" in kl:
                out["sm_max_mhz"] = v
    return out


def tensor_peak(pk, clocks, f16=False):
    """Useful peak of a split-precision conv timed inside a decode: the bf16
    figure x the nominal ratio of the MMA kind to bf16 (tf32 1.1 / 2.25; fp16
    1.0) / 3 products.  The burst figure applies when the timed region ran at
    the maximum SM clock with no power capping; under capping or a lower
    clock, the sustained figure scaled by the measured clock over the clock the
    sustained figure was taken at.  Returns (peak, source, burst peak).  The
    scaled figure never exceeds the burst figure: a clock near the maximum with
    a brief power cap takes the burst peak."""
    ratio = 1.0 if f16 else TF32_PER_BF16
    kind = (f"fp16/bf16 1.0 / 3 (3xF16)" if f16 else
            f"tf32/bf16 {TF32_PER_BF16:.3f} / 3 (3xTF32)")
    burst = pk["bf16"] * ratio / 3.0
    m = (clocks or {}).get("sm_mhz")
    mx = (clocks or {}).get("sm_max_mhz") or pk["sm_max_mhz"]
    capped = "sw_power_cap" in (clocks or {}).get("reasons", [])
    if m is None:
        return burst, f"{pk['source']} bf16 burst {pk['bf16']} TFLOP/s x {kind} (no clock samples)", burst
    if not capped and m >= 0.97 * mx:
        return burst, (f"{pk['source']} bf16 burst {pk['bf16']} TFLOP/s x {kind}; "
                       f"SM clock {m:.0f} of {mx:.0f} MHz, no power cap"), burst
    peak = pk["bf16_sustained"] * m / pk["sustained_mhz"] * ratio / 3.0
    if peak >= burst:
        return burst, (f"{pk['source']} bf16 burst {pk['bf16']} TFLOP/s x {kind}; "
                       f"SM clock {m:.0f} of {mx:.0f} MHz, "
                       f"power cap {'seen' if capped else 'not seen'} (the sustained figure "
                       f"scaled to this clock would exceed the burst figure)"), burst
    return peak, (f"{pk['source']} bf16 sustained {pk['bf16_sustained']} TFLOP/s at "
                  f"{pk['sustained_mhz']:.0f} MHz scaled to the measured {m:.0f} MHz, x {kind}; "
                  f"power cap {'seen' if capped else 'not seen'}"), \
        burst


# kernel classes on the tensor cores: 3xTF32, and the fp16 split
TENSOR_CLASSES = ("conv1d_tm", "conv1d_tc", "conv_transpose1d_tc", "conv_transpose1d_tm",
                  "conv1d_tm_f16", "conv_transpose1d_tm_f16")
F16_CLASSES = ("conv1d_tm_f16", "conv_transpose1d_tm_f16")

# Measured DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) over
# the algorithmic bytes, per kernel class, from one ncu capture of every launch
# of the class's kernel in one decode of the default workload; the bench's
# `traffic` is this ratio x the class's algorithmic bytes per launch.  A class
# whose kernel code changed since its capture has no entry (traffic null).
#   conv1d_tm_f16: the fp16-split conv1d_tm_kernel instances, all 180 AMP-conv
#   launches of one 60 s stereo decode, 35.52 GB against 42.01 GB algorithmic
#   (the algorithmic count takes the operand as 4 B per element; the two fp16
#   planes are 2 + 2 B); one ncu pass per launch.  The 3xTF32 class's last
#   capture predates the staged output loop: no entry.
NCU_TRAFFIC_RATIO = {"conv1d_tm_f16": 0.846}


def traffic_for(name, kd):
    r = NCU_TRAFFIC_RATIO.get(name)
    return None if r is None else r * kd["bytes"]


def roofline_for(name, kd, pk, clocks=None):
    """Achieved vs peak for one kernel class; achieved = algorithmic work per
    launch / average launch time (CUDA events on the launching stream)."""
    t = kd["avg_launch_ms"] / 1000.0
    if name in TENSOR_CLASSES:
        # useful FLOPs of the split conv; the tensor pipe issues 3 MMAs each
        peak, src, burst = tensor_peak(pk, clocks, f16=name in F16_CLASSES)
        ach = kd["flops"] / t / 1e12
        return {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                "frac": ach / peak, "frac_of_burst": ach / burst,
                "traffic": traffic_for(name, kd), "peak_source": src}
    mhz = (clocks or {}).get("sm_max_mhz") or pk["sm_max_mhz"]
    if kd["flops"] > 0:
        peak = SMS * FP32_LANES_PER_SM * 2 * mhz * 1e6 / 1e12
        ach = kd["flops"] / t / 1e12
        return {"bound": "alu", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                "frac": ach / peak, "traffic": traffic_for(name, kd),
                "peak_source": f"FP32 pipe: {SMS} SMs x {FP32_LANES_PER_SM} lanes x 2 x "
                               f"{mhz:.0f} MHz"}
    ach = kd["bytes"] / t / 1e9
    return {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": ach / pk["hbm_gbs"], "traffic": traffic_for(name, kd),
            "peak_source": f"{pk['source']} hbm_gbs"}


def host_cpu():
    """CPU model and logical core count of this host."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count()}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value, world, device):
    """The largest of every rank's `value` (each rank's device-timed total):
    the job takes as long as its slowest replica."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, audio_seconds_per_step, ms_per_step):
    """Whole-job audio-seconds per second: every replica decodes its own
    workload in the (max-over-ranks) step time."""
    return world * audio_seconds_per_step / (ms_per_step / 1000.0)


def cpu_baseline(workload, frames, steps=1):
    """The oracle as it stands, single-threaded, on a bounded sample: one side
    of the workload's decoder on its first `frames` latent frames."""
    import oracle
    z, params = workload.make()
    zs = np.ascontiguousarray(z[:1, :, :frames])
    oracle.decode(workload.geometry, params, zs)  # warm the library and caches
    times = []
    for _ in range(steps):
        t = time.perf_counter()
        oracle.decode(workload.geometry, params, zs)
        times.append(time.perf_counter() - t)
    audio = frames * workload.geometry.hop / workload.geometry.sample_rate
    return audio / statistics.mean(times), times, audio


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    w = synth.DECODER_WORKLOADS[args.workload]
    import oracle
    z, params = w.make()
    frames = 4
    zs = np.ascontiguousarray(z[:1, :, :frames])
    audio = frames * w.geometry.hop / w.geometry.sample_rate
    for _ in range(args.warmup):
        oracle.decode(w.geometry, params, zs)
    times = []
    for _ in range(args.steps):
        t = time.perf_counter()
        oracle.decode(w.geometry, params, zs)
        times.append(time.perf_counter() - t)
    value = audio / statistics.mean(times)
    sample = (f"oracle decode of one side, first {frames} latent frames "
              f"({audio:.3f} s of audio) of {w.name}")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * statistics.mean(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "frames": w.frames,
                   "tile_frames": w.tile_frames, "overlap_frames": w.overlap_frames,
                   "timed_sample": {"batch": 1, "frames": frames}},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample, **host_cpu()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_activation_sweep(args):
    """The activation over the sweep grid: per shape, W warm-up and K timed
    launches (CUDA events on the launching stream, L2 evicted between
    launches outside the events); achieved = 8 B per element / median time."""
    import torch
    from bigvgan_waveform_decoder_alias_b200 import native
    torch.cuda.set_device(0)
    pk = peaks()
    filt = torch.from_numpy(native.bv_filter_design()).cuda()
    flush = torch.empty(L2_FLUSH_BYTES // 4, device="cuda")
    B = 2
    rows = []
    with ClockSampler(0) as clk:
        for C, T in synth.ACT_SWEEP_GRID:
            # timing only: inputs of the workload's distribution drawn on the
            # device (the parity tests use the seeded host stream)
            g = torch.Generator(device="cuda").manual_seed(synth.ACT_SWEEP.seed)
            x = torch.randn((B, C, T), device="cuda", generator=g)
            la = torch.randn((C,), device="cuda", generator=g) * synth.SNAKE_STD
            lb = torch.randn((C,), device="cuda", generator=g) * synth.SNAKE_STD
            y = torch.empty_like(x)
            for _ in range(max(args.warmup, 3)):
                native.bv_activation1d(x, la, lb, filt, y=y)
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            for k in range(args.steps):
                flush.fill_(float(k))
                ev[k][0].record()
                native.bv_activation1d(x, la, lb, filt, y=y)
                ev[k][1].record()
            torch.cuda.synchronize()
            ms = statistics.median(a.elapsed_time(b) for a, b in ev)
            gbs = 8.0 * B * C * T / (ms / 1000) / 1e9
            rows.append({"C": C, "T": T, "ms": ms, "GB/s": gbs, "frac": gbs / pk["hbm_gbs"]})
            del x, y
    print(json.dumps({"mode": "activation_sweep", "batch": B, "unit": "GB/s",
                      "peak": pk["hbm_gbs"], "peak_source": f"{pk['source']} hbm_gbs",
                      "steps": args.steps, "warmup": args.warmup,
                      "l2": "evicted between launches (256 MiB write outside the events)",
                      "shapes": rows, "clocks": clk.summary()}), flush=True)
    return 0


def main():
    args = parse()
    world, rank, local = dist_init()
    if args.case:
        return run_case(args)
    if args.activation_sweep:
        return run_activation_sweep(args)
    if args.impl == "reference":
        return run_reference(args, world, rank)

    import torch
    import torch.distributed as dist
    from bigvgan_waveform_decoder_alias_b200 import native

    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    w = synth.DECODER_WORKLOADS[args.workload]
    z, params = w.make()
    if rank > 0:  # each replica decodes its own latent
        z = synth.NormalStream(w.seed + 1000 * rank).normal(z.shape, w.input_mean, w.input_std)
    dec = native.Decoder(w.geometry, params, tile_frames=w.tile_frames,
                         overlap_frames=w.overlap_frames, device=dev, tf32_only=args.tf32_only)
    # model load: the tensor-core weights split and packed once
    # (bv_decoder_prepare); every step decodes its own latent in full
    dec.prepare()
    zd = torch.from_numpy(z).to(dev)
    B, _, F = z.shape
    L = dec.output_length(F)
    y = torch.empty((B, w.geometry.out_channels, L), device=dev)
    ws = dec.workspace(B, F)
    flush = torch.empty(L2_FLUSH_BYTES // 4, device=dev)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(args.warmup, 3)):
        dec.decode(zd, y=y, workspace=ws)
    torch.cuda.synchronize()

    # ---------------------------------------------------------- timed region
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    n0 = native.launch_count()
    with ClockSampler(dev.index) as clk:
        for k in range(args.steps):
            flush.fill_(float(k))  # evict L2 between steps, outside the events
            ev[k][0].record(stream)
            dec.decode(zd, y=y, workspace=ws)
            ev[k][1].record(stream)
        torch.cuda.synchronize()
    barrier()
    launches = native.launch_count() - n0
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    ms_per_step = total_ms / args.steps
    audio_per_step = w.audio_seconds()
    value = job_throughput(world, audio_per_step, ms_per_step)
    y_check = y.detach().float()
    finite = bool(torch.isfinite(y_check).all().item())

    # ------------------- the same decode with every conv in 3xTF32, for scale
    tf32 = None
    if not args.tf32_only:
        dec32 = native.Decoder(w.geometry, params, tile_frames=w.tile_frames,
                               overlap_frames=w.overlap_frames, device=dev, tf32_only=True)
        dec32.prepare()
        y32 = torch.empty_like(y)
        for _ in range(max(args.warmup, 3)):
            dec32.decode(zd, y=y32, workspace=ws)
        torch.cuda.synchronize()
        ev3 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        barrier()
        with ClockSampler(dev.index) as clk32:
            for k in range(args.steps):
                flush.fill_(float(k))
                ev3[k][0].record(stream)
                dec32.decode(zd, y=y32, workspace=ws)
                ev3[k][1].record(stream)
            torch.cuda.synchronize()
        barrier()
        ms32 = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev3), world, dev) / args.steps
        # the two splits' outputs on the same latent (both against the oracle
        # in the golden tests)
        d = (y - y32).double()
        tf32 = {"value": job_throughput(world, audio_per_step, ms32), "unit": UNIT,
                "ms_per_step": ms32, "clocks": clk32.summary(),
                "rel_l2_vs_default": float(d.norm() / y32.double().norm())}
        del dec32, y32

    # -------------------------------------------- end to end through host memory
    zh = torch.from_numpy(z).pin_memory()
    yh = torch.empty((B, w.geometry.out_channels, L), dtype=torch.float32).pin_memory()
    wsh = dec.workspace(B, F, host=True)
    dec.decode_host(zh, yh, workspace=wsh)
    torch.cuda.synchronize()
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier()
    for k in range(args.steps):
        flush.fill_(float(k))
        ev2[k][0].record(stream)
        dec.decode_host(zh, yh, workspace=wsh)
        ev2[k][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev2), world, dev)
    e2e_value = job_throughput(world, audio_per_step, e2e_ms / args.steps)

    # ----------------------------------------- per-kernel timing (roofline)
    import ctypes
    Lb = native.lib()
    Lb.bv_timing_enable(1)
    Lb.bv_timing_reset()
    prof_steps = min(args.steps, 5)
    with ClockSampler(dev.index) as clk_prof:
        for k in range(prof_steps):
            flush.fill_(float(k))
            dec.decode(zd, y=y, workspace=ws)
        torch.cuda.synchronize()
    Stats = native.KernelStats * 16
    st = Stats()
    n = Lb.bv_timing_read(st, 16)
    Lb.bv_timing_enable(0)
    kernels = {}
    for i in range(max(n, 0)):
        s = st[i]
        kernels[s.name.decode()] = {"launches_per_step": s.launches / prof_steps,
                                    "ms_per_step": s.ms / prof_steps,
                                    "flops": s.flops / max(s.launches, 1),
                                    "bytes": s.bytes / max(s.launches, 1),
                                    "avg_launch_ms": s.ms / max(s.launches, 1)}
    pk = peaks()
    prof_clocks = clk_prof.summary()
    roofs = {name: roofline_for(name, kd, pk, prof_clocks) for name, kd in kernels.items()}
    for name, r in roofs.items():
        kernels[name]["roofline"] = r
    dom = max(kernels, key=lambda k: kernels[k]["ms_per_step"]) if kernels else None
    roof = dict(roofs[dom], kernel=dom) if dom else None
    # the fused activation, both forms (K1 writes [B, C, T]: 8 B per element;
    # K1tm writes the conv's hi/lo planes: 12 B): algorithmic bytes / time
    act_classes = [k for k in ("activation", "activation_tm") if k in kernels]
    acts = [kernels[k] for k in act_classes]
    act = None
    if acts:
        ms = sum(k["ms_per_step"] for k in acts)
        by = sum(k["bytes"] * k["launches_per_step"] for k in acts)
        gbs = by / (ms / 1000.0) / 1e9
        act = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
               "frac": gbs / pk["hbm_gbs"], "traffic": None,
               "peak_source": f"{pk['source']} hbm_gbs",
               "kernels": act_classes}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, times, audio = cpu_baseline(w, args.cpu_sample_frames)
        cpu = {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"oracle decode of one side, first {args.cpu_sample_frames} latent "
                         f"frames ({audio:.3f} s of audio) of {w.name}, "
                         f"{statistics.mean(times):.1f} s", **host_cpu()}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": w.name, "batch": B, "frames": F,
                       "audio_seconds_per_step": audio_per_step,
                       "sample_rate": w.geometry.sample_rate,
                       "l2": "flushed between steps (256 MiB write outside the timed events)",
                       "weights": "resident, split and ConvT packing prepared once at load",
                       "conv_split": ("3xTF32 throughout" if args.tf32_only else
                                      "fp16 split (3 products, fp32 accumulate) for the AMP "
                                      "and transposed convs of 48+ input channels in "
                                      "multiples of 8, 3xTF32 elsewhere"),
                       "parallelism": f"replicas x{world}"},
            "e2e": {"value": e2e_value, "unit": UNIT,
                    "h2d_bytes_per_step": int(zh.numel() * 4),
                    "d2h_bytes_per_step": int(yh.numel() * 4)},
            "gpu_launches": int(launches),
            "roofline": roof,
            "activation": act,
            "kernels": kernels,
            "cpu_baseline": cpu,
            "clocks": clk.summary(),
            "clocks_profiled_pass": prof_clocks,
            "output_finite": finite,
            "split_3xtf32": tf32,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
