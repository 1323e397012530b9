"""Seeded synthetic inputs: decoder geometries, workloads and random tensors.

This module holds shapes and random numbers only -- none of the decoder's
arithmetic.  The CUDA library and the parity oracle both consume the float32
arrays it produces.

Random numbers: SplitMix64 (Steele, Lea & Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014) used as a counter-based stream --
the i-th 64-bit word of stream ``seed`` is mix(seed + (i + 1) * 0x9E3779B97F4A7C15)
-- and the Box-Muller transform (Box & Muller 1958) on consecutive pairs of
words: u1 = ((w0 >> 11) + 1) / 2^53, u2 = (w1 >> 11) / 2^53,
n0 = sqrt(-2 ln u1) cos(2 pi u2), n1 = sqrt(-2 ln u1) sin(2 pi u2).
One stream per workload; the input is drawn first, then the parameters in
module order (``param_layout``), each tensor taking the next normals.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import List, Sequence, Tuple

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
M1 = np.uint64(0xBF58476D1CE4E5B9)
M2 = np.uint64(0x94D049BB133111EB)


def splitmix64_words(seed: int, start: int, count: int) -> np.ndarray:
    """Words start .. start+count-1 of SplitMix64 stream ``seed``."""
    i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed) + i * GAMMA
        z = (z ^ (z >> np.uint64(30))) * M1
        z = (z ^ (z >> np.uint64(27))) * M2
    return z ^ (z >> np.uint64(31))


class NormalStream:
    """Consecutive standard normals from one seeded SplitMix64 stream."""

    CHUNK = 1 << 22

    def __init__(self, seed: int):
        self.seed = int(seed)
        self.pos = 0  # index of the next normal

    def _normals(self, start: int, count: int) -> np.ndarray:
        # normals 2k and 2k+1 come from words 2k and 2k+1
        p0 = start // 2
        p1 = (start + count + 1) // 2
        w = splitmix64_words(self.seed, 2 * p0, 2 * (p1 - p0))
        u1 = ((w[0::2] >> np.uint64(11)) + np.uint64(1)).astype(np.float64) * 2.0 ** -53
        u2 = (w[1::2] >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
        r = np.sqrt(-2.0 * np.log(u1))
        th = 2.0 * np.pi * u2
        out = np.empty(2 * (p1 - p0), np.float64)
        out[0::2] = r * np.cos(th)
        out[1::2] = r * np.sin(th)
        off = start - 2 * p0
        return out[off:off + count]

    def normal(self, shape, mean=0.0, std=1.0) -> np.ndarray:
        n = int(np.prod(shape)) if len(shape) else 1
        out = np.empty(n, np.float32)
        done = 0
        while done < n:
            c = min(self.CHUNK, n - done)
            out[done:done + c] = (mean + std * self._normals(self.pos + done, c)).astype(np.float32)
            done += c
        self.pos += n
        return out.reshape(shape)


# ----------------------------------------------------------------- geometry


@dataclass(frozen=True)
class DecoderGeometry:
    """Shape of a BigVGAN-style decoder (conv_pre -> ConvT stages with AMP
    blocks averaged per stage -> act_post -> conv_post -> final op)."""
    in_channels: int
    pre_channels: int
    pre_kernel: int
    up_rates: Tuple[int, ...]
    up_kernels: Tuple[int, ...]
    up_channels: Tuple[int, ...]
    block_kernels: Tuple[int, ...]
    dilations: Tuple[int, ...]
    post_kernel: int
    out_channels: int
    final_act: str  # "none" | "clamp" | "tanh"
    sample_rate: int

    @property
    def hop(self) -> int:
        h = 1
        for r in self.up_rates:
            h *= r
        return h

    def replace(self, **kw) -> "DecoderGeometry":
        return dataclasses.replace(self, **kw)


def param_layout(g: DecoderGeometry) -> List[Tuple[str, Tuple[int, ...], str]]:
    """(name, shape, kind) of every decoder parameter in module order; kind is
    'w' (conv weight), 'b' (bias) or 'snake' (log alpha / log beta)."""
    out = []
    C = g.pre_channels
    out.append(("conv_pre.w", (C, g.in_channels, g.pre_kernel), "w"))
    out.append(("conv_pre.b", (C,), "b"))
    for i, (s, k, co) in enumerate(zip(g.up_rates, g.up_kernels, g.up_channels)):
        out.append((f"ups.{i}.w", (C, co, k), "w"))
        out.append((f"ups.{i}.b", (co,), "b"))
        C = co
        for j, kb in enumerate(g.block_kernels):
            for u, _d in enumerate(g.dilations):
                p = f"stage{i}.block{j}.unit{u}"
                out += [(f"{p}.act1.log_alpha", (C,), "snake"),
                        (f"{p}.act1.log_beta", (C,), "snake"),
                        (f"{p}.conv1.w", (C, C, kb), "w"),
                        (f"{p}.conv1.b", (C,), "b"),
                        (f"{p}.act2.log_alpha", (C,), "snake"),
                        (f"{p}.act2.log_beta", (C,), "snake"),
                        (f"{p}.conv2.w", (C, C, kb), "w"),
                        (f"{p}.conv2.b", (C,), "b")]
    out.append(("act_post.log_alpha", (C,), "snake"))
    out.append(("act_post.log_beta", (C,), "snake"))
    out.append(("conv_post.w", (g.out_channels, C, g.post_kernel), "w"))
    out.append(("conv_post.b", (g.out_channels,), "b"))
    return out


def param_count(g: DecoderGeometry) -> int:
    return int(sum(int(np.prod(s)) for _, s, _ in param_layout(g)))


# The parameter distributions of the synthetic decoders: conv and ConvT
# weights and biases N(0, 0.02), SnakeBeta log-alpha / log-beta N(0, 0.1).
WEIGHT_STD = 0.02
BIAS_STD = 0.02
SNAKE_STD = 0.1


def _draw_params(stream: NormalStream, layout) -> np.ndarray:
    total = sum(int(np.prod(s)) for _, s, _ in layout)
    flat = np.empty(total, np.float32)
    off = 0
    for _, shape, kind in layout:
        n = int(np.prod(shape))
        std = {"w": WEIGHT_STD, "b": BIAS_STD, "snake": SNAKE_STD}[kind]
        flat[off:off + n] = stream.normal((n,), 0.0, std)
        off += n
    return flat


# ---------------------------------------------------------------- workloads

H3 = DecoderGeometry(
    in_channels=32, pre_channels=1536, pre_kernel=7,
    up_rates=(5, 5, 2, 2, 2, 2, 2), up_kernels=(10, 10, 4, 4, 4, 4, 4),
    up_channels=(768, 384, 192, 96, 48, 24, 12),
    block_kernels=(3, 7, 11), dilations=(1, 3, 5),
    post_kernel=7, out_channels=1, final_act="tanh", sample_rate=32000)

LTX = DecoderGeometry(
    in_channels=64, pre_channels=1024, pre_kernel=7,
    up_rates=(5, 2, 2, 2, 2, 2), up_kernels=(10, 4, 4, 4, 4, 4),
    up_channels=(512, 256, 128, 64, 32, 16),
    block_kernels=(3, 7, 11), dilations=(1, 3, 5),
    post_kernel=7, out_channels=1, final_act="clamp", sample_rate=16000)


@dataclass(frozen=True)
class DecoderWorkload:
    name: str
    geometry: DecoderGeometry
    batch: int
    frames: int
    seed: int
    input_mean: float = 0.0
    input_std: float = 1.0
    tile_frames: int = 0
    overlap_frames: int = 0

    def audio_seconds(self) -> float:
        """Seconds of audio per side (stereo counts once)."""
        return self.frames * self.geometry.hop / self.geometry.sample_rate

    def make(self):
        """(z [B, in_ch, frames], flat params) drawn from this workload's seed."""
        s = NormalStream(self.seed)
        z = s.normal((self.batch, self.geometry.in_channels, self.frames),
                     self.input_mean, self.input_std)
        return z, _draw_params(s, param_layout(self.geometry))


@dataclass(frozen=True)
class AmpWorkload:
    name: str
    batch: int
    channels: int
    length: int
    kernel: int
    dilations: Tuple[int, ...]
    seed: int

    def layout(self):
        C, K = self.channels, self.kernel
        out = []
        for u, _ in enumerate(self.dilations):
            out += [(f"unit{u}.act1.log_alpha", (C,), "snake"),
                    (f"unit{u}.act1.log_beta", (C,), "snake"),
                    (f"unit{u}.conv1.w", (C, C, K), "w"), (f"unit{u}.conv1.b", (C,), "b"),
                    (f"unit{u}.act2.log_alpha", (C,), "snake"),
                    (f"unit{u}.act2.log_beta", (C,), "snake"),
                    (f"unit{u}.conv2.w", (C, C, K), "w"), (f"unit{u}.conv2.b", (C,), "b")]
        return out

    def make(self):
        s = NormalStream(self.seed)
        x = s.normal((self.batch, self.channels, self.length))
        return x, _draw_params(s, self.layout())


@dataclass(frozen=True)
class ActivationWorkload:
    name: str
    batch: int
    channels: int
    length: int
    seed: int

    def make(self):
        s = NormalStream(self.seed)
        x = s.normal((self.batch, self.channels, self.length))
        la = s.normal((self.channels,), 0.0, SNAKE_STD)
        lb = s.normal((self.channels,), 0.0, SNAKE_STD)
        return x, la, lb


AMP_BLOCK_C32 = AmpWorkload("amp_block_c32_t8192", 1, 32, 8192, 3, (1, 3, 5), seed=0)
ACT_SWEEP = ActivationWorkload("activation_c512_t65536", 2, 512, 65536, seed=1)
ACT_SWEEP_GRID = [(c, t) for c in (64, 128, 256, 512, 768, 1024, 1536)
                  for t in (4096, 16384, 65536, 262144)]
H3_10S = DecoderWorkload("h3_decoder_10s_stereo", H3, 2, 400, seed=2)
LTX_VOCODER = DecoderWorkload("ltx_vocoder_500f_stereo", LTX, 2, 500, seed=3,
                              input_mean=-4.0, input_std=2.0)
H3_60S_TILED = DecoderWorkload("h3_decoder_60s_stereo_tiled", H3, 2, 2400, seed=4,
                               tile_frames=200, overlap_frames=16)

DECODER_WORKLOADS = {w.name: w for w in (H3_10S, LTX_VOCODER, H3_60S_TILED)}


# ------------------------------------------ LTX bandwidth-extension tail
# The extender's mel front end reads two buffers from its checkpoint (the
# STFT's DFT x window bases and the mel filterbank); none is available here,
# so they are synthesised as the reference's preprocessing builds them.


def stft_basis(n_fft: int) -> np.ndarray:
    """[2 n_freqs, n_fft] float32, n_freqs = n_fft/2 + 1: rows w[j]
    cos(2 pi r j / n_fft), then -w[j] sin(2 pi r j / n_fft), w the periodic
    Hann window 0.5 - 0.5 cos(2 pi j / n_fft) (a one-sided DFT of the
    windowed frame)."""
    j = np.arange(n_fft)
    w = 0.5 - 0.5 * np.cos(2 * np.pi * j / n_fft)
    r = np.arange(n_fft // 2 + 1)[:, None]
    ang = 2 * np.pi * r * j[None, :] / n_fft
    return np.concatenate([w * np.cos(ang), -w * np.sin(ang)]).astype(np.float32)


def slaney_mel_basis(sample_rate: int, n_fft: int, n_mels: int, fmin: float,
                     fmax: float) -> np.ndarray:
    """[n_mels, n_fft/2 + 1] float32 triangular filters on the Slaney mel
    scale (linear 3 f / 200 below 1 kHz, logarithmic above, 27 mels per
    factor 6.4), each scaled by 2 / (upper edge - lower edge) in Hz (Slaney's
    area normalisation)."""
    f_min_log, min_log_mel, logstep = 1000.0, 15.0, np.log(6.4) / 27.0

    def hz_to_mel(f):
        f = np.asarray(f, np.float64)
        return np.where(f >= f_min_log, min_log_mel + np.log(np.maximum(f, 1e-12) / f_min_log)
                        / logstep, 3.0 * f / 200.0)

    def mel_to_hz(m):
        m = np.asarray(m, np.float64)
        return np.where(m >= min_log_mel, f_min_log * np.exp(logstep * (m - min_log_mel)),
                        200.0 * m / 3.0)

    freqs = np.linspace(0, sample_rate / 2, n_fft // 2 + 1)
    pts = mel_to_hz(np.linspace(hz_to_mel(fmin), hz_to_mel(fmax), n_mels + 2))
    lower = (freqs[None, :] - pts[:-2, None]) / (pts[1:-1] - pts[:-2])[:, None]
    upper = (pts[2:, None] - freqs[None, :]) / (pts[2:] - pts[1:-1])[:, None]
    fb = np.maximum(0.0, np.minimum(lower, upper))
    fb *= (2.0 / (pts[2:] - pts[:-2]))[:, None]
    return fb.astype(np.float32)


@dataclass(frozen=True)
class BweSpec:
    """The extender's mel front end and rates: n_fft-sample frames every
    `hop` samples, n_mels bins over [fmin, fmax] at the input rate, output
    rate = ratio x input rate."""
    in_rate: int
    ratio: int
    n_fft: int
    hop: int
    n_mels: int
    fmin: float
    fmax: float

    def bases(self):
        return (stft_basis(self.n_fft),
                slaney_mel_basis(self.in_rate, self.n_fft, self.n_mels, self.fmin, self.fmax))


LTX_BWE_SPEC = BweSpec(in_rate=16000, ratio=3, n_fft=512, hop=80, n_mels=64, fmin=0.0,
                       fmax=8000.0)

# The extender generator: BigVGAN v2 on the folded stereo log-mel (2 x 64
# channels in, 2 out), rates 6, 5, 2, 2, 2 (240 = 3 x the mel hop), no final
# op (its output is a residual added to the upsampled input).
LTX_BWE = DecoderGeometry(
    in_channels=128, pre_channels=512, pre_kernel=7,
    up_rates=(6, 5, 2, 2, 2), up_kernels=(12, 10, 4, 4, 4),
    up_channels=(256, 128, 64, 32, 16),
    block_kernels=(3, 7, 11), dilations=(1, 3, 5),
    post_kernel=7, out_channels=2, final_act="none", sample_rate=48000)


# ------------------------------------------------ Music-3 DAV decoder


@dataclass(frozen=True)
class DavGeometry:
    """Shape of a MiniMax-Music-3 DAV decoder: dec_in (one tap) -> conv_pre ->
    stages of plain Snake, ConvT and residual units at the given dilations
    -> Snake -> conv_post -> final op."""
    latent_channels: int
    in_channels: int
    pre_channels: int
    pre_kernel: int
    up_rates: Tuple[int, ...]
    up_kernels: Tuple[int, ...]
    up_channels: Tuple[int, ...]
    dilations: Tuple[int, ...]
    unit_kernel: int
    post_kernel: int
    out_channels: int
    final_act: str
    sample_rate: int

    @property
    def hop(self) -> int:
        h = 1
        for r in self.up_rates:
            h *= r
        return h

    def replace(self, **kw) -> "DavGeometry":
        return dataclasses.replace(self, **kw)


def dav_param_layout(g: DavGeometry) -> List[Tuple[str, Tuple[int, ...], str]]:
    """(name, shape, kind) of every DAV parameter in module order; kind
    'alpha' is a plain Snake's alpha, used as stored."""
    out = [("dec_in.w", (g.in_channels, g.latent_channels, 1), "w"),
           ("dec_in.b", (g.in_channels,), "b"),
           ("conv_pre.w", (g.pre_channels, g.in_channels, g.pre_kernel), "w"),
           ("conv_pre.b", (g.pre_channels,), "b")]
    C = g.pre_channels
    for i, (k, co) in enumerate(zip(g.up_kernels, g.up_channels)):
        out += [(f"stage{i}.act.alpha", (C,), "alpha"),
                (f"stage{i}.up.w", (C, co, k), "w"), (f"stage{i}.up.b", (co,), "b")]
        C = co
        for u, _d in enumerate(g.dilations):
            p = f"stage{i}.unit{u}"
            out += [(f"{p}.a1.alpha", (C,), "alpha"),
                    (f"{p}.c1.w", (C, C, g.unit_kernel), "w"), (f"{p}.c1.b", (C,), "b"),
                    (f"{p}.a2.alpha", (C,), "alpha"),
                    (f"{p}.c2.w", (C, C, 1), "w"), (f"{p}.c2.b", (C,), "b")]
    out += [("act_post.alpha", (C,), "alpha"),
            ("conv_post.w", (g.out_channels, C, g.post_kernel), "w"),
            ("conv_post.b", (g.out_channels,), "b")]
    return out


def dav_param_count(g: DavGeometry) -> int:
    return int(sum(int(np.prod(s)) for _, s, _ in dav_param_layout(g)))


# Plain Snake alpha of the synthetic DAV decoders: 1 + N(0, 0.1), used as
# stored (the layers' initial value plus spread).
ALPHA_MEAN = 1.0
ALPHA_STD = 0.1


def draw_dav_params(stream: "NormalStream", g: DavGeometry) -> np.ndarray:
    layout = dav_param_layout(g)
    flat = np.empty(sum(int(np.prod(s)) for _, s, _ in layout), np.float32)
    off = 0
    for _, shape, kind in layout:
        n = int(np.prod(shape))
        if kind == "alpha":
            flat[off:off + n] = stream.normal((n,), ALPHA_MEAN, ALPHA_STD)
        else:
            flat[off:off + n] = stream.normal((n,), 0.0, WEIGHT_STD if kind == "w" else BIAS_STD)
        off += n
    return flat


# A DAC-style channel plan for Music-3's DAV decoder (strides 8, 8, 4, 2,
# dilations 1, 3, 9, 7-tap convs, tanh, 44.1 kHz; the 128-channel latent is a
# stereo pair of 64): decoder width 1536 halving per stage.
MUSIC3_DAV = DavGeometry(
    latent_channels=64, in_channels=64, pre_channels=1536, pre_kernel=7,
    up_rates=(8, 8, 4, 2), up_kernels=(16, 16, 8, 4), up_channels=(768, 384, 192, 96),
    dilations=(1, 3, 9), unit_kernel=7, post_kernel=7, out_channels=1, final_act="tanh",
    sample_rate=44100)


def tiny_dav_geometry(**kw) -> DavGeometry:
    """A small DAV decoder with the same structure, for oracle-speed tests."""
    base = DavGeometry(
        latent_channels=8, in_channels=8, pre_channels=48, pre_kernel=7,
        up_rates=(4, 2, 2), up_kernels=(8, 4, 4), up_channels=(32, 16, 8),
        dilations=(1, 3, 9), unit_kernel=7, post_kernel=7, out_channels=1, final_act="tanh",
        sample_rate=44100)
    return base.replace(**kw)


def tiny_geometry(**kw) -> DecoderGeometry:
    """A small decoder with the same structure, for tests the oracle runs in
    seconds (both stride parities, several blocks and dilations)."""
    base = DecoderGeometry(
        in_channels=8, pre_channels=48, pre_kernel=7,
        up_rates=(5, 2, 2), up_kernels=(10, 4, 4), up_channels=(32, 16, 8),
        block_kernels=(3, 7, 11), dilations=(1, 3, 5),
        post_kernel=7, out_channels=1, final_act="tanh", sample_rate=32000)
    return base.replace(**kw)
