"""Parity oracle for the BigVGAN alias-free decoder (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the bench's CPU-baseline
leg may import this package.  It is a plain single-threaded C statement of
the decoder (``bv_oracle.c``) that accumulates in double, loaded through
ctypes; it shares nothing with the CUDA library.

Functions take and return numpy float32 arrays in [B, C, T] layout.  The
decoder geometry is passed as a mapping or an object with the attributes
``in_channels, pre_channels, pre_kernel, up_rates, up_kernels, up_channels,
block_kernels, dilations, post_kernel, out_channels, final_act``.

Sources: docs.rs cortiq-engine 0.5.74 ``audiovae.rs`` (MiniMax-H3 BigVGAN),
0.6.3 ``ltxaudio.rs`` (LTX-2.5 BigVGAN v2), 0.5.89 ``music3.rs`` (windowing).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i32p = ctypes.POINTER(ctypes.c_int)

FINAL_ACTS = {"none": 0, "clamp": 1, "tanh": 2}


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.orc_bessel_i0.restype = ctypes.c_double
        L.orc_bessel_i0.argtypes = [ctypes.c_double]
        L.orc_sinc.restype = ctypes.c_double
        L.orc_sinc.argtypes = [ctypes.c_double]
        L.orc_kaiser_sinc.argtypes = [ctypes.c_double, ctypes.c_double, ctypes.c_int, _f64p]
        L.orc_activation1d.argtypes = [_f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       _f32p, _f32p, _f32p, _f32p, ctypes.c_int,
                                       ctypes.c_double, ctypes.c_int, _f32p]
        L.orc_conv1d.argtypes = [_f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _f32p,
                                 _f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                 ctypes.c_int, ctypes.c_int, _f32p]
        L.orc_conv_transpose1d.argtypes = L.orc_conv1d.argtypes
        L.orc_latent_front_end.argtypes = [_f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           _f32p, _f32p, _f32p, _f32p, ctypes.c_int,
                                           ctypes.c_int, _f32p]
        L.orc_conv1d_points.argtypes = [_f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        _f32p, _f32p, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_int, _i64p, ctypes.c_int,
                                        _f64p]
        L.orc_conv_transpose1d_points.argtypes = L.orc_conv1d_points.argtypes
        L.orc_activation1d_points.argtypes = [_f32p, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, _f32p, _f32p, _f32p, _f32p,
                                              ctypes.c_int, ctypes.c_double, _i64p,
                                              ctypes.c_int, _f64p]
        L.orc_amp_block.argtypes = [_f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _f32p,
                                    ctypes.c_int, _i32p, ctypes.c_int, _f32p, _f32p,
                                    ctypes.c_int, ctypes.c_double, ctypes.c_int, _f32p]
        L.orc_decoder_param_count.restype = ctypes.c_long
        L.orc_decoder_param_count.argtypes = [_i32p]
        L.orc_decoder_hop.restype = ctypes.c_long
        L.orc_decoder_hop.argtypes = [_i32p]
        L.orc_decoder_raw_len.restype = ctypes.c_long
        L.orc_decoder_raw_len.argtypes = [_i32p, ctypes.c_int]
        L.orc_decode.argtypes = [_i32p, _f32p, _f32p, ctypes.c_int, ctypes.c_int, _f32p,
                                 _f32p, ctypes.c_int, ctypes.c_double, ctypes.c_int, _f32p]
        L.orc_decode_tiled.argtypes = [_i32p, _f32p, _f32p, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, _f32p, _f32p, ctypes.c_int,
                                       ctypes.c_double, ctypes.c_int, _f32p, _f32p]
        L.orc_tile_count.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.orc_snake1d.argtypes = [_f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _f32p,
                                  ctypes.c_int, _f32p]
        L.orc_mel_stft.argtypes = [_f32p, ctypes.c_int, ctypes.c_int, _f32p, ctypes.c_int,
                                   ctypes.c_int, ctypes.c_int, _f32p, ctypes.c_int,
                                   ctypes.c_int, _f32p]
        L.orc_mel_frames.restype = ctypes.c_long
        L.orc_mel_frames.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.orc_hann_sinc_upsample.argtypes = [_f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, _f32p]
        L.orc_bwe_tail.argtypes = [_i32p, _f32p, _f32p, ctypes.c_int, ctypes.c_int, _f32p,
                                   ctypes.c_int, ctypes.c_int, ctypes.c_int, _f32p,
                                   ctypes.c_int, ctypes.c_int, _f32p, _f32p, ctypes.c_int,
                                   ctypes.c_int, _f32p]
        L.orc_dav_param_count.restype = ctypes.c_long
        L.orc_dav_param_count.argtypes = [_i32p]
        L.orc_dav_hop.restype = ctypes.c_long
        L.orc_dav_hop.argtypes = [_i32p]
        L.orc_dav_decode.argtypes = [_i32p, _f32p, _f32p, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, _f32p]
        _LIB = L
    return _LIB


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _p32(a):
    return None if a is None else a.ctypes.data_as(_f32p)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


# ------------------------------------------------------------------ filter


def bessel_i0(x: float) -> float:
    return lib().orc_bessel_i0(float(x))


def sinc(x: float) -> float:
    return lib().orc_sinc(float(x))


def kaiser_sinc_f64(cutoff=0.25, half_width=0.3, k=12) -> np.ndarray:
    out = np.zeros(k, np.float64)
    _check(lib().orc_kaiser_sinc(cutoff, half_width, k, out.ctypes.data_as(_f64p)),
           "kaiser_sinc")
    return out


def kaiser_sinc(cutoff=0.25, half_width=0.3, k=12) -> np.ndarray:
    """The designed filter as the pages hand it out: float taps."""
    return kaiser_sinc_f64(cutoff, half_width, k).astype(np.float32)


# ------------------------------------------------------------------ layers


def activation1d(x, log_alpha, log_beta, up=None, down=None, eps=1e-9, store_f64=False):
    x = _f32(x)
    B, C, T = x.shape
    up = kaiser_sinc() if up is None else _f32(up)
    down = up if down is None else _f32(down)
    la, lb = _f32(log_alpha), _f32(log_beta)
    y = np.empty_like(x)
    _check(lib().orc_activation1d(_p32(x), B, C, T, _p32(la), _p32(lb), _p32(up),
                                  _p32(down), len(up), eps, int(store_f64), _p32(y)),
           "activation1d")
    return y


def conv1d(x, w, bias, dilation=1, pad=None, store_f64=False):
    x, w = _f32(x), _f32(w)
    B, Cin, T = x.shape
    Cout, Cin2, K = w.shape
    assert Cin2 == Cin
    if pad is None:
        pad = (K * dilation - dilation) // 2
    Tout = T + 2 * pad - dilation * (K - 1)
    b = None if bias is None else _f32(bias)
    y = np.empty((B, Cout, Tout), np.float32)
    _check(lib().orc_conv1d(_p32(x), B, Cin, T, _p32(w), _p32(b), Cout, K, dilation,
                            pad, int(store_f64), _p32(y)), "conv1d")
    return y


def latent_front_end(z, mean, std, w, bias, store_f64=False):
    """[H3] ``AudioVae::decode`` front end: normalised latents z [C, S, T]
    (stereo: S = 2) -> per side z std + mean, then ``dec_in_proj`` (one-tap
    conv, w [Cout, C, 1]) -> [S, Cout, T]."""
    z, w = _f32(z), _f32(w)
    C, S, T = z.shape
    Cout, C2, K = w.shape
    assert C2 == C and K == 1
    b = None if bias is None else _f32(bias)
    out = np.empty((S, Cout, T), np.float32)
    _check(lib().orc_latent_front_end(_p32(z), C, S, T, _p32(_f32(mean)), _p32(_f32(std)),
                                      _p32(w), _p32(b), Cout, int(store_f64), _p32(out)),
           "latent_front_end")
    return out


def conv_transpose1d(x, w, bias, stride, pad=None, store_f64=False):
    x, w = _f32(x), _f32(w)
    B, Cin, T = x.shape
    Cin2, Cout, K = w.shape
    assert Cin2 == Cin
    if pad is None:
        pad = (K - stride) // 2
    Tout = (T - 1) * stride + K - 2 * pad
    b = None if bias is None else _f32(bias)
    y = np.empty((B, Cout, Tout), np.float32)
    _check(lib().orc_conv_transpose1d(_p32(x), B, Cin, T, _p32(w), _p32(b), Cout, K,
                                      stride, pad, int(store_f64), _p32(y)),
           "conv_transpose1d")
    return y


def _idx(points):
    idx = np.ascontiguousarray(np.asarray(points, dtype=np.int64).reshape(-1, 3))
    return idx, idx.shape[0]


def conv1d_points(x, w, bias, dilation, pad, points):
    x, w = _f32(x), _f32(w)
    B, Cin, T = x.shape
    Cout, _, K = w.shape
    b = None if bias is None else _f32(bias)
    idx, n = _idx(points)
    out = np.empty(n, np.float64)
    _check(lib().orc_conv1d_points(_p32(x), B, Cin, T, _p32(w), _p32(b), Cout, K,
                                   dilation, pad, idx.ctypes.data_as(_i64p), n,
                                   out.ctypes.data_as(_f64p)), "conv1d_points")
    return out


def conv_transpose1d_points(x, w, bias, stride, pad, points):
    x, w = _f32(x), _f32(w)
    B, Cin, T = x.shape
    _, Cout, K = w.shape
    b = None if bias is None else _f32(bias)
    idx, n = _idx(points)
    out = np.empty(n, np.float64)
    _check(lib().orc_conv_transpose1d_points(_p32(x), B, Cin, T, _p32(w), _p32(b), Cout,
                                             K, stride, pad, idx.ctypes.data_as(_i64p), n,
                                             out.ctypes.data_as(_f64p)),
           "conv_transpose1d_points")
    return out


def activation1d_points(x, log_alpha, log_beta, points, up=None, down=None, eps=1e-9):
    x = _f32(x)
    B, C, T = x.shape
    up = kaiser_sinc() if up is None else _f32(up)
    down = up if down is None else _f32(down)
    la, lb = _f32(log_alpha), _f32(log_beta)
    idx, n = _idx(points)
    out = np.empty(n, np.float64)
    _check(lib().orc_activation1d_points(_p32(x), B, C, T, _p32(la), _p32(lb), _p32(up),
                                         _p32(down), len(up), eps,
                                         idx.ctypes.data_as(_i64p), n,
                                         out.ctypes.data_as(_f64p)), "activation1d_points")
    return out


def amp_block(x, params, kernel_size, dilations, filt=None, eps=1e-9, store_f64=False):
    """One AMP block; `params` flat in the block's module order."""
    x, params = _f32(x), _f32(params)
    B, C, T = x.shape
    d = np.ascontiguousarray(np.asarray(dilations, np.int32))
    need = len(d) * (4 * C + 2 * (C * C * kernel_size + C))
    if params.size != need:
        raise ValueError(f"amp block params: {params.size} values, need {need}")
    f = kaiser_sinc() if filt is None else _f32(filt)
    y = np.empty_like(x)
    _check(lib().orc_amp_block(_p32(x), B, C, T, _p32(params), kernel_size,
                               d.ctypes.data_as(_i32p), len(d), _p32(f), _p32(f), len(f), eps,
                               int(store_f64), _p32(y)), "amp_block")
    return y


# ----------------------------------------------------------------- decoder


def _get(geo, name):
    return geo[name] if isinstance(geo, dict) else getattr(geo, name)


def geometry_ints(geo) -> np.ndarray:
    g = np.zeros(41, np.int32)
    rates, upk, upch = (list(_get(geo, n)) for n in ("up_rates", "up_kernels", "up_channels"))
    bk, dil = list(_get(geo, "block_kernels")), list(_get(geo, "dilations"))
    fa = _get(geo, "final_act")
    g[0], g[1], g[2], g[3] = (_get(geo, "in_channels"), _get(geo, "pre_channels"),
                              _get(geo, "pre_kernel"), len(rates))
    g[4:4 + len(rates)] = rates
    g[12:12 + len(upk)] = upk
    g[20:20 + len(upch)] = upch
    g[28] = len(bk)
    g[29:29 + len(bk)] = bk
    g[33] = len(dil)
    g[34:34 + len(dil)] = dil
    g[38], g[39] = _get(geo, "post_kernel"), _get(geo, "out_channels")
    g[40] = FINAL_ACTS[fa] if isinstance(fa, str) else int(fa)
    return g


def param_count(geo) -> int:
    g = geometry_ints(geo)
    n = lib().orc_decoder_param_count(g.ctypes.data_as(_i32p))
    if n < 0:
        raise ValueError("bad decoder geometry")
    return int(n)


def hop(geo) -> int:
    g = geometry_ints(geo)
    return int(lib().orc_decoder_hop(g.ctypes.data_as(_i32p)))


def raw_len(geo, frames) -> int:
    g = geometry_ints(geo)
    return int(lib().orc_decoder_raw_len(g.ctypes.data_as(_i32p), int(frames)))


def decode(geo, params, z, filt=None, eps=1e-9, store_f64=False):
    """z [B, in_ch, frames] -> waveform [B, out_ch, frames * hop]."""
    g = geometry_ints(geo)
    z, params = _f32(z), _f32(params)
    if params.size != param_count(geo):
        raise ValueError(f"params has {params.size} values, geometry needs {param_count(geo)}")
    B, _, F = z.shape
    f = kaiser_sinc() if filt is None else _f32(filt)
    y = np.empty((B, int(g[39]), F * hop(geo)), np.float32)
    _check(lib().orc_decode(g.ctypes.data_as(_i32p), _p32(params), _p32(z), B, F,
                            _p32(f), _p32(f), len(f), eps, int(store_f64), _p32(y)),
           "decode")
    return y


def tile_count(frames, tile, overlap) -> int:
    return int(lib().orc_tile_count(int(frames), int(tile), int(overlap)))


def decode_tiled(geo, params, z, tile, overlap, tiles=None, filt=None, eps=1e-9,
                 store_f64=False):
    """Tiled decode; ``tiles=(lo, hi)`` restricts which tiles are decoded (the
    samples no chosen tile covers come back as NaN).  Returns (y, count)."""
    g = geometry_ints(geo)
    z, params = _f32(z), _f32(params)
    B, _, F = z.shape
    lo, hi = (0, tile_count(F, tile, overlap)) if tiles is None else tiles
    f = kaiser_sinc() if filt is None else _f32(filt)
    L = F * hop(geo)
    y = np.empty((B, int(g[39]), L), np.float32)
    cnt = np.empty(L, np.float32)
    _check(lib().orc_decode_tiled(g.ctypes.data_as(_i32p), _p32(params), _p32(z), B, F,
                                  tile, overlap, lo, hi, _p32(f), _p32(f), len(f), eps,
                                  int(store_f64), _p32(y), _p32(cnt)), "decode_tiled")
    return y, cnt


# ------------------------------------------------------- Music-3 DAV decoder


def snake1d(x, alpha, store_f64=False):
    """Plain Snake, alpha used as stored: x + sin^2(alpha x) / (alpha + 1e-9)
    (the audiovae.rs page's `Snake`)."""
    x = _f32(x)
    B, C, T = x.shape
    y = np.empty_like(x)
    _check(lib().orc_snake1d(_p32(x), B, C, T, _p32(_f32(alpha)), int(store_f64), _p32(y)),
           "snake1d")
    return y


def dav_geometry_ints(geo) -> np.ndarray:
    g = np.zeros(38, np.int32)
    rates, upk, upch = (list(_get(geo, n)) for n in ("up_rates", "up_kernels", "up_channels"))
    dil = list(_get(geo, "dilations"))
    fa = _get(geo, "final_act")
    g[0], g[1], g[2], g[3], g[4] = (_get(geo, "latent_channels"), _get(geo, "in_channels"),
                                    _get(geo, "pre_channels"), _get(geo, "pre_kernel"),
                                    len(rates))
    g[5:5 + len(rates)] = rates
    g[13:13 + len(upk)] = upk
    g[21:21 + len(upch)] = upch
    g[29] = len(dil)
    g[30:30 + len(dil)] = dil
    g[34], g[35], g[36] = (_get(geo, "unit_kernel"), _get(geo, "post_kernel"),
                           _get(geo, "out_channels"))
    g[37] = FINAL_ACTS[fa] if isinstance(fa, str) else int(fa)
    return g


def dav_param_count(geo) -> int:
    g = dav_geometry_ints(geo)
    return int(lib().orc_dav_param_count(g.ctypes.data_as(_i32p)))


def dav_hop(geo) -> int:
    g = dav_geometry_ints(geo)
    return int(lib().orc_dav_hop(g.ctypes.data_as(_i32p)))


def dav_decode(geo, params, z, store_f64=False):
    """MiniMax-Music-3 DAV decoder (the audiovae.rs page's `Music3Dav`):
    z [B, latent_channels, frames] -> [B, out_channels, frames * hop]; the
    page's 128-channel stereo latent is B = 2 halves of 64."""
    g = dav_geometry_ints(geo)
    z, params = _f32(z), _f32(params)
    if params.size != dav_param_count(geo):
        raise ValueError(f"params has {params.size} values, geometry needs "
                         f"{dav_param_count(geo)}")
    B, _, F = z.shape
    y = np.empty((B, int(g[36]), F * dav_hop(geo)), np.float32)
    _check(lib().orc_dav_decode(g.ctypes.data_as(_i32p), _p32(params), _p32(z), B, F,
                                int(store_f64), _p32(y)), "dav_decode")
    return y


# --------------------------------------------- LTX bandwidth-extension tail


def mel_frames(T, n_fft, hop) -> int:
    return int(lib().orc_mel_frames(int(T), int(n_fft), int(hop)))


def mel_stft(x, basis, mel_basis, hop, store_f64=False):
    """The ltxaudio.rs page's causal log-mel (`MelStft::forward`): x [C, T],
    basis [2 n_freqs, n_fft], mel_basis [n_mels, n_freqs] -> the folded
    [C n_mels, frames] the extender reads."""
    x, basis, mel_basis = _f32(x), _f32(basis), _f32(mel_basis)
    C, T = x.shape
    nf2, L = basis.shape
    n_mels, nf = mel_basis.shape
    assert nf2 == 2 * nf
    frames = mel_frames(T, L, hop)
    out = np.empty((C * n_mels, frames), np.float32)
    _check(lib().orc_mel_stft(_p32(x), C, T, _p32(basis), nf, L, hop, _p32(mel_basis), n_mels,
                              int(store_f64), _p32(out)), "mel_stft")
    return out


def hann_sinc_upsample(x, ratio, store_f64=False):
    """The ltxaudio.rs page's `hann_sinc_upsample`: x [C, T] -> [C, ratio T]."""
    x = _f32(x)
    C, T = x.shape
    y = np.empty((C, ratio * T), np.float32)
    _check(lib().orc_hann_sinc_upsample(_p32(x), C, T, ratio, int(store_f64), _p32(y)),
           "hann_sinc_upsample")
    return y


def bwe_tail(geo, params, low, basis, mel_basis, hop, ratio, filt=None, store_f64=False):
    """The ltxaudio.rs page's `AudioStack::decode_from_mel` after the first
    generator: low [C, T] -> clamp(extender(log-mel(low)) + upsample(low)),
    [C, ratio T]."""
    g = geometry_ints(geo)
    low, params = _f32(low), _f32(params)
    basis, mel_basis = _f32(basis), _f32(mel_basis)
    C, T = low.shape
    nf2, L = basis.shape
    n_mels, nf = mel_basis.shape
    f = kaiser_sinc() if filt is None else _f32(filt)
    y = np.empty((C, ratio * T), np.float32)
    _check(lib().orc_bwe_tail(g.ctypes.data_as(_i32p), _p32(params), _p32(low), C, T,
                              _p32(basis), nf, L, hop, _p32(mel_basis), n_mels, ratio, _p32(f),
                              _p32(f), len(f), int(store_f64), _p32(y)), "bwe_tail")
    return y
