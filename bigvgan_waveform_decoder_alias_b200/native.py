"""ctypes binding of libbv.so (the C ABI declared in include/bv.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libbv.  PyTorch provides device memory and streams.  There is no
fallback: if libbv.so cannot be loaded, or a call fails, a BVError is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np
import torch

from .synth import DecoderGeometry

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbv.so")

BV_FILTER_TAPS = 12
BV_MAX_UP = 8
BV_MAX_BLOCKS = 4
BV_MAX_DIL = 4
FINAL_ACTS = {"none": 0, "clamp": 1, "tanh": 2}
STATUS = {0: "BV_OK", 1: "BV_ERR_ARG", 2: "BV_ERR_SHAPE", 3: "BV_ERR_WORKSPACE",
          4: "BV_ERR_CUDA", 5: "BV_ERR_TIMEOUT", 6: "BV_ERR_UNSUPPORTED",
          7: "BV_ERR_RANGE"}


class BVError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


_fp = ctypes.c_void_p


class Epilogue(ctypes.Structure):
    _fields_ = [("residual", _fp), ("scale", ctypes.c_float), ("accumulate", ctypes.c_int),
                ("final_act", ctypes.c_int)]


class AmpParams(ctypes.Structure):
    _fields_ = [("kernel_size", ctypes.c_int), ("n_dilations", ctypes.c_int),
                ("dilation", ctypes.c_int * BV_MAX_DIL),
                ("conv1_w", _fp * BV_MAX_DIL), ("conv1_b", _fp * BV_MAX_DIL),
                ("conv2_w", _fp * BV_MAX_DIL), ("conv2_b", _fp * BV_MAX_DIL),
                ("act_log_alpha", _fp * (2 * BV_MAX_DIL)),
                ("act_log_beta", _fp * (2 * BV_MAX_DIL)),
                ("up_filter", _fp), ("down_filter", _fp)]


class DecoderConfig(ctypes.Structure):
    _fields_ = [("in_channels", ctypes.c_int), ("pre_channels", ctypes.c_int),
                ("pre_kernel", ctypes.c_int), ("n_up", ctypes.c_int),
                ("up_rate", ctypes.c_int * BV_MAX_UP), ("up_kernel", ctypes.c_int * BV_MAX_UP),
                ("up_channels", ctypes.c_int * BV_MAX_UP), ("n_blocks", ctypes.c_int),
                ("block_kernel", ctypes.c_int * BV_MAX_BLOCKS), ("n_dilations", ctypes.c_int),
                ("dilation", ctypes.c_int * BV_MAX_DIL), ("post_kernel", ctypes.c_int),
                ("out_channels", ctypes.c_int), ("final_act", ctypes.c_int),
                ("tile_frames", ctypes.c_int), ("overlap_frames", ctypes.c_int),
                ("latent_channels", ctypes.c_int), ("tf32_only", ctypes.c_int)]


class DecoderWeights(ctypes.Structure):
    _fields_ = [("pre_w", _fp), ("pre_b", _fp),
                ("up_w", _fp * BV_MAX_UP), ("up_b", _fp * BV_MAX_UP),
                ("amp", (AmpParams * BV_MAX_BLOCKS) * BV_MAX_UP),
                ("post_log_alpha", _fp), ("post_log_beta", _fp),
                ("post_w", _fp), ("post_b", _fp),
                ("up_filter", _fp), ("down_filter", _fp),
                ("latents_mean", _fp), ("latents_std", _fp),
                ("dec_in_w", _fp), ("dec_in_b", _fp), ("prepared", _fp)]


class DavConfig(ctypes.Structure):
    _fields_ = [("latent_channels", ctypes.c_int), ("in_channels", ctypes.c_int),
                ("pre_channels", ctypes.c_int), ("pre_kernel", ctypes.c_int),
                ("n_up", ctypes.c_int), ("up_rate", ctypes.c_int * BV_MAX_UP),
                ("up_kernel", ctypes.c_int * BV_MAX_UP),
                ("up_channels", ctypes.c_int * BV_MAX_UP), ("n_dilations", ctypes.c_int),
                ("dilation", ctypes.c_int * BV_MAX_DIL), ("unit_kernel", ctypes.c_int),
                ("post_kernel", ctypes.c_int), ("out_channels", ctypes.c_int),
                ("final_act", ctypes.c_int)]


class DavWeights(ctypes.Structure):
    _fields_ = [("dec_in_w", _fp), ("dec_in_b", _fp), ("pre_w", _fp), ("pre_b", _fp),
                ("stage_alpha", _fp * BV_MAX_UP), ("up_w", _fp * BV_MAX_UP),
                ("up_b", _fp * BV_MAX_UP),
                ("a1", (_fp * BV_MAX_DIL) * BV_MAX_UP), ("c1_w", (_fp * BV_MAX_DIL) * BV_MAX_UP),
                ("c1_b", (_fp * BV_MAX_DIL) * BV_MAX_UP),
                ("a2", (_fp * BV_MAX_DIL) * BV_MAX_UP), ("c2_w", (_fp * BV_MAX_DIL) * BV_MAX_UP),
                ("c2_b", (_fp * BV_MAX_DIL) * BV_MAX_UP),
                ("post_alpha", _fp), ("post_w", _fp), ("post_b", _fp)]


class KernelStats(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_uint64),
                ("ms", ctypes.c_double), ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


_LIB = None


def lib():
    """Load libbv.so; raises if it is missing (no fallback exists)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise BVError(4, f"{LIB_PATH} is missing: build it with "
                         "`python -m bigvgan_waveform_decoder_alias_b200.build_native`")
    L = ctypes.CDLL(LIB_PATH)
    c_int, c_float, c_double, c_size = ctypes.c_int, ctypes.c_float, ctypes.c_double, ctypes.c_size_t
    L.bv_last_error.restype = ctypes.c_char_p
    L.bv_version.restype = ctypes.c_char_p
    L.bv_launch_count.restype = ctypes.c_uint64
    L.bv_sync_status.argtypes = [_fp]
    L.bv_debug_set_wait_limit.restype = ctypes.c_longlong
    L.bv_debug_set_wait_limit.argtypes = [ctypes.c_longlong]
    L.bv_timing_enable.argtypes = [c_int]
    L.bv_timing_enable.restype = None
    L.bv_timing_reset.argtypes = []
    L.bv_timing_reset.restype = None
    L.bv_timing_read.argtypes = [ctypes.POINTER(KernelStats), c_int]
    L.bv_timing_read.restype = c_int
    L.bv_filter_design.argtypes = [c_double, c_double, c_int, ctypes.POINTER(c_float)]
    L.bv_activation1d.argtypes = [_fp, _fp, c_int, c_int, c_int, _fp, _fp, _fp, _fp, c_float, _fp]
    L.bv_sin_squared.argtypes = [_fp, _fp, ctypes.c_int64, _fp]
    L.bv_conv1d.argtypes = [_fp, c_int, c_int, c_int, _fp, _fp, c_int, c_int, c_int, c_int,
                            ctypes.POINTER(Epilogue), _fp, _fp]
    L.bv_conv_transpose1d.argtypes = [_fp, c_int, c_int, c_int, _fp, _fp, c_int, c_int, c_int,
                                      c_int, _fp, _fp]
    L.bv_act_conv1d_workspace_size.restype = c_size
    L.bv_act_conv1d_workspace_size.argtypes = [c_int] * 6
    L.bv_act_conv1d.argtypes = [_fp, c_int, c_int, c_int, _fp, _fp, _fp, _fp, c_float, _fp, _fp,
                                c_int, c_int, c_int, c_int, ctypes.POINTER(Epilogue), _fp, _fp,
                                c_size, _fp]
    L.bv_conv_transpose1d_workspace_size.restype = c_size
    L.bv_conv_transpose1d_workspace_size.argtypes = [c_int] * 6
    L.bv_conv_transpose1d_ws.argtypes = [_fp, c_int, c_int, c_int, _fp, _fp, c_int, c_int,
                                         c_int, c_int, _fp, _fp, c_size, _fp]
    L.bv_amp_block_workspace_size.restype = c_size
    L.bv_amp_block_workspace_size.argtypes = [c_int, c_int, c_int]
    L.bv_amp_block_workspace_size_tc.restype = c_size
    L.bv_amp_block_workspace_size_tc.argtypes = [c_int, c_int, c_int, ctypes.POINTER(AmpParams)]
    L.bv_amp_block.argtypes = [_fp, c_int, c_int, c_int, ctypes.POINTER(AmpParams), _fp, c_float,
                               c_int, _fp, c_size, _fp]
    L.bv_amp_block_static.argtypes = [_fp, c_int, c_int, c_int, ctypes.POINTER(AmpParams), _fp,
                                      c_float, c_int, _fp]
    L.bv_latent_front_end.argtypes = [_fp, c_int, c_int, c_int, _fp, _fp, _fp, _fp, c_int, _fp,
                                      _fp]
    L.bv_decoder_param_count.restype = ctypes.c_int64
    L.bv_decoder_param_count.argtypes = [ctypes.POINTER(DecoderConfig)]
    L.bv_decoder_weights_from_flat.argtypes = [ctypes.POINTER(DecoderConfig), _fp, _fp, _fp,
                                               ctypes.POINTER(DecoderWeights)]
    L.bv_decoder_output_length.restype = ctypes.c_int64
    L.bv_decoder_output_length.argtypes = [ctypes.POINTER(DecoderConfig), c_int]
    L.bv_decode_workspace_size.restype = c_size
    L.bv_decode_workspace_size.argtypes = [ctypes.POINTER(DecoderConfig), c_int, c_int]
    L.bv_decode.argtypes = [ctypes.POINTER(DecoderConfig), ctypes.POINTER(DecoderWeights), _fp,
                            c_int, c_int, _fp, _fp, c_size, _fp]
    L.bv_decoder_prepared_size.restype = c_size
    L.bv_decoder_prepared_size.argtypes = [ctypes.POINTER(DecoderConfig)]
    L.bv_decoder_prepare.argtypes = [ctypes.POINTER(DecoderConfig), ctypes.POINTER(DecoderWeights),
                                     _fp, c_size, _fp]
    L.bv_decode_workspace_size_prepared.restype = c_size
    L.bv_decode_workspace_size_prepared.argtypes = [ctypes.POINTER(DecoderConfig), c_int, c_int]
    L.bv_decoder_tile_count.restype = c_int
    L.bv_decoder_tile_count.argtypes = [ctypes.POINTER(DecoderConfig), c_int]
    L.bv_decoder_unit_length.restype = ctypes.c_int64
    L.bv_decoder_unit_length.argtypes = [ctypes.POINTER(DecoderConfig), c_int]
    L.bv_decode_units_workspace_size.restype = c_size
    L.bv_decode_units_workspace_size.argtypes = [ctypes.POINTER(DecoderConfig), c_int, c_int,
                                                 ctypes.c_int64, ctypes.c_int64]
    L.bv_decode_units.argtypes = [ctypes.POINTER(DecoderConfig), ctypes.POINTER(DecoderWeights),
                                  _fp, c_int, c_int, ctypes.c_int64, ctypes.c_int64, _fp, _fp,
                                  c_size, _fp]
    L.bv_stitch_units.argtypes = [ctypes.POINTER(DecoderConfig), c_int, c_int, _fp, _fp, _fp]
    L.bv_mel_frames.restype = ctypes.c_int64
    L.bv_mel_frames.argtypes = [c_int, c_int, c_int]
    L.bv_mel_stft.argtypes = [_fp, c_int, c_int, _fp, c_int, c_int, c_int, _fp, c_int, _fp, _fp]
    L.bv_sinc_upsample.argtypes = [_fp, c_int, c_int, c_int, _fp, _fp]
    L.bv_bwe_tail_workspace_size.restype = c_size
    L.bv_bwe_tail_workspace_size.argtypes = [ctypes.POINTER(DecoderConfig), c_int, c_int, c_int,
                                             c_int, c_int, c_int]
    L.bv_bwe_tail.argtypes = [ctypes.POINTER(DecoderConfig), ctypes.POINTER(DecoderWeights), _fp,
                              c_int, c_int, _fp, c_int, c_int, _fp, c_int, c_int, _fp, _fp,
                              c_size, _fp]
    L.bv_dav_param_count.restype = ctypes.c_int64
    L.bv_dav_param_count.argtypes = [ctypes.POINTER(DavConfig)]
    L.bv_dav_weights_from_flat.argtypes = [ctypes.POINTER(DavConfig), _fp,
                                           ctypes.POINTER(DavWeights)]
    L.bv_dav_output_length.restype = ctypes.c_int64
    L.bv_dav_output_length.argtypes = [ctypes.POINTER(DavConfig), c_int]
    L.bv_dav_workspace_size.restype = c_size
    L.bv_dav_workspace_size.argtypes = [ctypes.POINTER(DavConfig), c_int, c_int]
    L.bv_dav_decode.argtypes = [ctypes.POINTER(DavConfig), ctypes.POINTER(DavWeights), _fp, c_int,
                                c_int, _fp, _fp, c_size, _fp]
    L.bv_decode_host_workspace_size.restype = c_size
    L.bv_decode_host_workspace_size.argtypes = [ctypes.POINTER(DecoderConfig), c_int, c_int]
    L.bv_decode_host.argtypes = [ctypes.POINTER(DecoderConfig), ctypes.POINTER(DecoderWeights),
                                 _fp, c_int, c_int, _fp, _fp, c_size, _fp]
    _LIB = L
    return L


def _check(status: int):
    if status != 0:
        raise BVError(status, lib().bv_last_error().decode(errors="replace"))


def last_error() -> str:
    return lib().bv_last_error().decode(errors="replace")


def version() -> str:
    return lib().bv_version().decode()


def launch_count() -> int:
    return int(lib().bv_launch_count())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
        raise BVError(1, "tensors must be contiguous float32 CUDA tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def timing(enable: bool):
    lib().bv_timing_enable(int(bool(enable)))


def timing_reset():
    lib().bv_timing_reset()


def timing_read(max_classes: int = 16) -> dict:
    buf = (KernelStats * max_classes)()
    n = lib().bv_timing_read(buf, max_classes)
    if n < 0:
        raise BVError(4, "bv_timing_read failed")
    return {buf[i].name.decode(): {"launches": int(buf[i].launches), "ms": buf[i].ms,
                                   "flops": buf[i].flops, "bytes": buf[i].bytes}
            for i in range(min(n, max_classes))}


def sync_status(stream=None):
    _check(lib().bv_sync_status(_stream(stream)))


def set_wait_limit(polls: int) -> int:
    """Testing hook: polls after which the tensor-core kernels' bounded waits
    give up (negative restores the default); returns the previous value."""
    return int(lib().bv_debug_set_wait_limit(int(polls)))


# ------------------------------------------------------------------ layers


def bv_filter_design(cutoff=0.25, half_width=0.3, taps=BV_FILTER_TAPS) -> np.ndarray:
    out = np.zeros(taps, np.float32)
    _check(lib().bv_filter_design(cutoff, half_width, taps,
                                  out.ctypes.data_as(ctypes.POINTER(ctypes.c_float))))
    return out


def bv_activation1d(x, log_alpha, log_beta, up_filter, down_filter=None, eps=1e-9, y=None,
                    stream=None):
    B, C, T = x.shape
    down_filter = up_filter if down_filter is None else down_filter
    y = torch.empty_like(x) if y is None else y
    _check(lib().bv_activation1d(_ptr(x), _ptr(y), B, C, T, _ptr(log_alpha), _ptr(log_beta),
                                 _ptr(up_filter), _ptr(down_filter), eps, _stream(stream)))
    return y


def bv_sin_squared(z, out=None, stream=None):
    out = torch.empty_like(z) if out is None else out
    _check(lib().bv_sin_squared(_ptr(z), _ptr(out), z.numel(), _stream(stream)))
    return out


def bv_conv1d(x, w, bias, dilation=1, pad=None, residual=None, scale=1.0, accumulate=False,
              final_act=0, y=None, stream=None):
    B, Cin, T = x.shape
    Cout, _, K = w.shape
    pad = (K * dilation - dilation) // 2 if pad is None else pad
    Tout = T + 2 * pad - dilation * (K - 1)
    y = torch.empty((B, Cout, Tout), device=x.device, dtype=torch.float32) if y is None else y
    ep = Epilogue(_ptr(residual), float(scale), int(bool(accumulate)),
                  FINAL_ACTS.get(final_act, final_act) if isinstance(final_act, str) else int(final_act))
    _check(lib().bv_conv1d(_ptr(x), B, Cin, T, _ptr(w), _ptr(bias), Cout, K, dilation, pad,
                           ctypes.byref(ep), _ptr(y), _stream(stream)))
    return y


def bv_conv_transpose1d(x, w, bias, stride, pad=None, y=None, stream=None):
    B, Cin, T = x.shape
    _, Cout, K = w.shape
    pad = (K - stride) // 2 if pad is None else pad
    Tout = (T - 1) * stride + K - 2 * pad
    y = torch.empty((B, Cout, Tout), device=x.device, dtype=torch.float32) if y is None else y
    _check(lib().bv_conv_transpose1d(_ptr(x), B, Cin, T, _ptr(w), _ptr(bias), Cout, K, stride,
                                     pad, _ptr(y), _stream(stream)))
    return y


def _epilogue(residual, scale, accumulate, final_act) -> Epilogue:
    fa = FINAL_ACTS.get(final_act, final_act) if isinstance(final_act, str) else int(final_act)
    return Epilogue(_ptr(residual), float(scale), int(bool(accumulate)), fa)


def bv_act_conv1d(x, log_alpha, log_beta, up_filter, w, bias, dilation=1, pad=None,
                  down_filter=None, eps=1e-9, residual=None, scale=1.0, accumulate=False,
                  final_act=0, y=None, workspace=None, stream=None):
    """Activation then conv on the decoder's own kernels (time-major tensor
    cores where the shape qualifies)."""
    B, C, T = x.shape
    Cout, _, K = w.shape
    pad = (K * dilation - dilation) // 2 if pad is None else pad
    Tout = T + 2 * pad - dilation * (K - 1)
    down_filter = up_filter if down_filter is None else down_filter
    y = torch.empty((B, Cout, Tout), device=x.device, dtype=torch.float32) if y is None else y
    need = int(lib().bv_act_conv1d_workspace_size(B, C, T, Cout, K, dilation))
    if workspace is None:
        workspace = torch.empty(need // 4 + 64, device=x.device, dtype=torch.float32)
    ep = _epilogue(residual, scale, accumulate, final_act)
    _check(lib().bv_act_conv1d(_ptr(x), B, C, T, _ptr(log_alpha), _ptr(log_beta),
                               _ptr(up_filter), _ptr(down_filter), eps, _ptr(w), _ptr(bias),
                               Cout, K, dilation, pad, ctypes.byref(ep), _ptr(y),
                               _ptr(workspace), workspace.numel() * 4, _stream(stream)))
    return y


def bv_conv_transpose1d_ws(x, w, bias, stride, pad=None, y=None, workspace=None, stream=None):
    """ConvTranspose1d on the decoder's own kernels (given a workspace)."""
    B, Cin, T = x.shape
    _, Cout, K = w.shape
    pad = (K - stride) // 2 if pad is None else pad
    Tout = (T - 1) * stride + K - 2 * pad
    y = torch.empty((B, Cout, Tout), device=x.device, dtype=torch.float32) if y is None else y
    need = int(lib().bv_conv_transpose1d_workspace_size(B, Cin, T, Cout, K, stride))
    if workspace is None:
        workspace = torch.empty(need // 4 + 64, device=x.device, dtype=torch.float32)
    _check(lib().bv_conv_transpose1d_ws(_ptr(x), B, Cin, T, _ptr(w), _ptr(bias), Cout, K, stride,
                                        pad, _ptr(y), _ptr(workspace), workspace.numel() * 4,
                                        _stream(stream)))
    return y


def bv_latent_front_end(z, mean, std, w, bias=None, out=None, stream=None):
    """Normalised latents z [C, S, T] -> [S, Cout, T] (de-normalise, then
    the one-tap dec_in projection w [Cout, C, 1])."""
    C, S, T = z.shape
    Cout = w.shape[0]
    out = torch.empty((S, Cout, T), device=z.device, dtype=torch.float32) if out is None else out
    _check(lib().bv_latent_front_end(_ptr(z), C, S, T, _ptr(mean), _ptr(std), _ptr(w),
                                     _ptr(bias), Cout, _ptr(out), _stream(stream)))
    return out


def amp_params(kernel_size: int, dilations: Sequence[int], tensors: dict, up_filter,
               down_filter=None) -> AmpParams:
    """AmpParams from tensors named unit{u}.{act1,act2}.log_{alpha,beta} and
    unit{u}.{conv1,conv2}.{w,b} (the order of synth.AmpWorkload.layout)."""
    p = AmpParams()
    p.kernel_size = kernel_size
    p.n_dilations = len(dilations)
    for u, d in enumerate(dilations):
        p.dilation[u] = d
        p.conv1_w[u] = _ptr(tensors[f"unit{u}.conv1.w"])
        p.conv1_b[u] = _ptr(tensors.get(f"unit{u}.conv1.b"))
        p.conv2_w[u] = _ptr(tensors[f"unit{u}.conv2.w"])
        p.conv2_b[u] = _ptr(tensors.get(f"unit{u}.conv2.b"))
        p.act_log_alpha[2 * u] = _ptr(tensors[f"unit{u}.act1.log_alpha"])
        p.act_log_beta[2 * u] = _ptr(tensors[f"unit{u}.act1.log_beta"])
        p.act_log_alpha[2 * u + 1] = _ptr(tensors[f"unit{u}.act2.log_alpha"])
        p.act_log_beta[2 * u + 1] = _ptr(tensors[f"unit{u}.act2.log_beta"])
    p.up_filter = _ptr(up_filter)
    p.down_filter = _ptr(up_filter if down_filter is None else down_filter)
    return p


def bv_amp_block_workspace_size(B, C, T) -> int:
    return int(lib().bv_amp_block_workspace_size(B, C, T))


def bv_amp_block_workspace_size_tc(B, C, T, params: AmpParams) -> int:
    return int(lib().bv_amp_block_workspace_size_tc(B, C, T, ctypes.byref(params)))


def bv_amp_block(x, params: AmpParams, y=None, scale=1.0, accumulate=False, workspace=None,
                 stream=None, keepalive=None, tensor_core=True):
    """tensor_core: size a new workspace for the time-major tensor-core path
    (taken by the block's qualifying convs); False keeps every conv on
    [B, C, T] operands."""
    B, C, T = x.shape
    y = torch.empty_like(x) if y is None else y
    need = (bv_amp_block_workspace_size_tc(B, C, T, params) if tensor_core
            else bv_amp_block_workspace_size(B, C, T))
    if workspace is None:
        workspace = torch.empty(need // 4 + 64, device=x.device, dtype=torch.float32)
    _check(lib().bv_amp_block(_ptr(x), B, C, T, ctypes.byref(params), _ptr(y), float(scale),
                              int(bool(accumulate)), _ptr(workspace), workspace.numel() * 4,
                              _stream(stream)))
    return y


# ----------------------------------------------------------------- decoder


def decoder_config(g: DecoderGeometry, tile_frames=0, overlap_frames=0,
                   tf32_only=False) -> DecoderConfig:
    c = DecoderConfig()
    c.in_channels, c.pre_channels, c.pre_kernel = g.in_channels, g.pre_channels, g.pre_kernel
    c.n_up = len(g.up_rates)
    for i, (s, k, ch) in enumerate(zip(g.up_rates, g.up_kernels, g.up_channels)):
        c.up_rate[i], c.up_kernel[i], c.up_channels[i] = s, k, ch
    c.n_blocks = len(g.block_kernels)
    for j, k in enumerate(g.block_kernels):
        c.block_kernel[j] = k
    c.n_dilations = len(g.dilations)
    for u, d in enumerate(g.dilations):
        c.dilation[u] = d
    c.post_kernel, c.out_channels = g.post_kernel, g.out_channels
    c.final_act = FINAL_ACTS[g.final_act] if isinstance(g.final_act, str) else int(g.final_act)
    c.tile_frames, c.overlap_frames = tile_frames, overlap_frames
    c.tf32_only = int(bool(tf32_only))
    return c


def bv_decoder_param_count(cfg: DecoderConfig) -> int:
    return int(lib().bv_decoder_param_count(ctypes.byref(cfg)))


class Decoder:
    """A decoder bound to device-resident weights: the library's public entry
    for whole decodes.  `params` is the flat parameter vector (module order),
    `filt` the 12 resampling taps (both filters)."""

    def __init__(self, geometry: DecoderGeometry, params, filt=None, tile_frames=0,
                 overlap_frames=0, device="cuda", front_end=None, tf32_only=False):
        """front_end: optional (latents_mean, latents_std, dec_in_w, dec_in_b)
        of the latent front end; decode() then takes normalised latents
        [latent_channels, B, frames].  tf32_only: every tensor-core conv in
        3xTF32 (else the AMP convs that qualify use the fp16 split)."""
        self.geometry = geometry
        self.cfg = decoder_config(geometry, tile_frames, overlap_frames, tf32_only)
        n = bv_decoder_param_count(self.cfg)
        if n < 0:
            raise BVError(2, last_error())
        params = torch.as_tensor(params, dtype=torch.float32)
        if params.numel() != n:
            raise BVError(2, f"params has {params.numel()} values, the geometry needs {n}")
        self.params = params.to(device).contiguous()
        if filt is None:
            filt = bv_filter_design(0.25, 0.3, BV_FILTER_TAPS)
        self.filt = torch.as_tensor(np.asarray(filt, np.float32)).to(device).contiguous()
        self.weights = DecoderWeights()
        _check(lib().bv_decoder_weights_from_flat(ctypes.byref(self.cfg), _ptr(self.params),
                                                  _ptr(self.filt), _ptr(self.filt),
                                                  ctypes.byref(self.weights)))
        self.front_end = None
        if front_end is not None:
            mean, std, w, b = (None if a is None else
                               torch.as_tensor(a, dtype=torch.float32).to(device).contiguous()
                               for a in front_end)
            self.front_end = (mean, std, w, b)  # keeps the pointed-to memory alive
            self.cfg.latent_channels = int(w.shape[1])
            self.weights.latents_mean, self.weights.latents_std = _ptr(mean), _ptr(std)
            self.weights.dec_in_w, self.weights.dec_in_b = _ptr(w), _ptr(b)
        self.device = self.params.device
        self._ws = None

    def output_length(self, frames: int) -> int:
        return int(lib().bv_decoder_output_length(ctypes.byref(self.cfg), frames))

    def prepare(self, stream=None):
        """Split and pack the tensor-core weights once into a buffer the
        later decodes read (bv_decoder_prepare)."""
        n = int(lib().bv_decoder_prepared_size(ctypes.byref(self.cfg)))
        self._prepared = torch.empty(n // 4 + 64, device=self.device, dtype=torch.float32)
        self.weights.prepared = None
        _check(lib().bv_decoder_prepare(ctypes.byref(self.cfg), ctypes.byref(self.weights),
                                        _ptr(self._prepared), self._prepared.numel() * 4,
                                        _stream(stream)))
        self.weights.prepared = _ptr(self._prepared)
        self._ws = None
        return self

    def workspace_size(self, B: int, frames: int, host=False) -> int:
        if self.weights.prepared and not host:
            n = int(lib().bv_decode_workspace_size_prepared(ctypes.byref(self.cfg), B, frames))
            if n == 0:
                raise BVError(2, last_error())
            return n
        f = lib().bv_decode_host_workspace_size if host else lib().bv_decode_workspace_size
        n = int(f(ctypes.byref(self.cfg), B, frames))
        if n == 0:
            raise BVError(2, last_error())
        return n

    def workspace(self, B: int, frames: int, host=False) -> torch.Tensor:
        need = self.workspace_size(B, frames, host)
        if self._ws is None or self._ws.numel() * 4 < need:
            self._ws = torch.empty(need // 4 + 64, device=self.device, dtype=torch.float32)
        return self._ws

    def _bf(self, z):
        """(B, frames) of a decode input: [B, C, F], or [C, B, F] latents."""
        if self.cfg.latent_channels > 0:
            return z.shape[1], z.shape[2]
        return z.shape[0], z.shape[2]

    def decode(self, z: torch.Tensor, y=None, workspace=None, stream=None) -> torch.Tensor:
        B, F = self._bf(z)
        L = self.output_length(F)
        y = torch.empty((B, self.cfg.out_channels, L), device=z.device, dtype=torch.float32) \
            if y is None else y
        ws = self.workspace(B, F) if workspace is None else workspace
        _check(lib().bv_decode(ctypes.byref(self.cfg), ctypes.byref(self.weights), _ptr(z), B, F,
                               _ptr(y), _ptr(ws), ws.numel() * 4, _stream(stream)))
        return y

    # ------------------------------------------------ units, for sharding
    def tile_count(self, frames: int) -> int:
        return int(lib().bv_decoder_tile_count(ctypes.byref(self.cfg), frames))

    def unit_length(self, frames: int) -> int:
        return int(lib().bv_decoder_unit_length(ctypes.byref(self.cfg), frames))

    def decode_units(self, z: torch.Tensor, unit_begin: int, unit_end: int, y_units=None,
                     workspace=None, stream=None) -> torch.Tensor:
        """Units [unit_begin, unit_end) (unit k B + b: tile k of side b) ->
        rows [unit_end - unit_begin, out_channels, unit_length]."""
        B, F = self._bf(z)
        if y_units is None:
            y_units = torch.empty((unit_end - unit_begin, self.cfg.out_channels,
                                   self.unit_length(F)), device=z.device, dtype=torch.float32)
        if workspace is None:
            need = int(lib().bv_decode_units_workspace_size(ctypes.byref(self.cfg), B, F,
                                                            unit_begin, unit_end))
            if need == 0:
                raise BVError(2, last_error())
            workspace = torch.empty(need // 4 + 64, device=z.device, dtype=torch.float32)
        _check(lib().bv_decode_units(ctypes.byref(self.cfg), ctypes.byref(self.weights), _ptr(z),
                                     B, F, unit_begin, unit_end, _ptr(y_units), _ptr(workspace),
                                     workspace.numel() * 4, _stream(stream)))
        return y_units

    def stitch_units(self, y_units: torch.Tensor, B: int, frames: int, y=None,
                     stream=None) -> torch.Tensor:
        """All tiles x B unit rows in unit order -> y [B, out_channels, frames hop]."""
        if y is None:
            y = torch.empty((B, self.cfg.out_channels, self.output_length(frames)),
                            device=y_units.device, dtype=torch.float32)
        _check(lib().bv_stitch_units(ctypes.byref(self.cfg), B, frames, _ptr(y_units), _ptr(y),
                                     _stream(stream)))
        return y

    def decode_host(self, z_host: torch.Tensor, y_host: torch.Tensor, workspace=None,
                    stream=None):
        """Host (pinned) latent in, host waveform out; asynchronous on the stream."""
        if z_host.is_cuda or y_host.is_cuda:
            raise BVError(1, "decode_host takes host tensors")
        B, F = self._bf(z_host)
        ws = self.workspace(B, F, host=True) if workspace is None else workspace
        _check(lib().bv_decode_host(ctypes.byref(self.cfg), ctypes.byref(self.weights),
                                    ctypes.c_void_p(z_host.data_ptr()), B, F,
                                    ctypes.c_void_p(y_host.data_ptr()), _ptr(ws),
                                    ws.numel() * 4, _stream(stream)))
        return y_host


# ------------------------------------------------------- Music-3 DAV decoder


def dav_config(g) -> DavConfig:
    c = DavConfig()
    c.latent_channels, c.in_channels = g.latent_channels, g.in_channels
    c.pre_channels, c.pre_kernel = g.pre_channels, g.pre_kernel
    c.n_up = len(g.up_rates)
    for i, (r, k, ch) in enumerate(zip(g.up_rates, g.up_kernels, g.up_channels)):
        c.up_rate[i], c.up_kernel[i], c.up_channels[i] = r, k, ch
    c.n_dilations = len(g.dilations)
    for u, d in enumerate(g.dilations):
        c.dilation[u] = d
    c.unit_kernel, c.post_kernel, c.out_channels = g.unit_kernel, g.post_kernel, g.out_channels
    c.final_act = FINAL_ACTS[g.final_act] if isinstance(g.final_act, str) else int(g.final_act)
    return c


class DavDecoder:
    """The MiniMax-Music-3 DAV decoder bound to device-resident weights
    (flat parameter vector in module order)."""

    def __init__(self, geometry, params, device="cuda"):
        self.geometry = geometry
        self.cfg = dav_config(geometry)
        n = int(lib().bv_dav_param_count(ctypes.byref(self.cfg)))
        if n < 0:
            raise BVError(2, last_error())
        params = torch.as_tensor(params, dtype=torch.float32)
        if params.numel() != n:
            raise BVError(2, f"params has {params.numel()} values, the geometry needs {n}")
        self.params = params.to(device).contiguous()
        self.weights = DavWeights()
        _check(lib().bv_dav_weights_from_flat(ctypes.byref(self.cfg), _ptr(self.params),
                                              ctypes.byref(self.weights)))
        self._ws = None

    def output_length(self, frames: int) -> int:
        return int(lib().bv_dav_output_length(ctypes.byref(self.cfg), frames))

    def workspace(self, B: int, frames: int) -> torch.Tensor:
        need = int(lib().bv_dav_workspace_size(ctypes.byref(self.cfg), B, frames))
        if need == 0:
            raise BVError(2, last_error())
        if self._ws is None or self._ws.numel() * 4 < need:
            self._ws = torch.empty(need // 4 + 64, device=self.params.device,
                                   dtype=torch.float32)
        return self._ws

    def decode(self, z: torch.Tensor, y=None, workspace=None, stream=None) -> torch.Tensor:
        B, _, F = z.shape
        y = torch.empty((B, self.cfg.out_channels, self.output_length(F)), device=z.device,
                        dtype=torch.float32) if y is None else y
        ws = self.workspace(B, F) if workspace is None else workspace
        _check(lib().bv_dav_decode(ctypes.byref(self.cfg), ctypes.byref(self.weights), _ptr(z),
                                   B, F, _ptr(y), _ptr(ws), ws.numel() * 4, _stream(stream)))
        return y


# ----------------------------------------------- bandwidth-extension tail


def bv_mel_stft(x, basis, mel_basis, hop, out=None, stream=None):
    """x [C, T] -> folded log-mel [C n_mels, frames]."""
    C, T = x.shape
    nf2, L = basis.shape
    n_mels = mel_basis.shape[0]
    frames = int(lib().bv_mel_frames(T, L, hop))
    out = torch.empty((C * n_mels, frames), device=x.device, dtype=torch.float32) \
        if out is None else out
    _check(lib().bv_mel_stft(_ptr(x), C, T, _ptr(basis), nf2 // 2, L, hop, _ptr(mel_basis),
                             n_mels, _ptr(out), _stream(stream)))
    return out


def bv_sinc_upsample(x, ratio, y=None, stream=None):
    C, T = x.shape
    y = torch.empty((C, ratio * T), device=x.device, dtype=torch.float32) if y is None else y
    _check(lib().bv_sinc_upsample(_ptr(x), C, T, ratio, _ptr(y), _stream(stream)))
    return y


class BweTail:
    """The bandwidth-extension tail: an extender decoder (a DecoderGeometry
    with its flat parameters) and its mel front end (synth.BweSpec bases)."""

    def __init__(self, geometry, params, spec, basis, mel_basis, filt=None, device="cuda"):
        self.dec = Decoder(geometry, params, filt=filt, device=device)
        self.spec = spec
        self.basis = torch.as_tensor(basis, dtype=torch.float32).to(device).contiguous()
        self.mel_basis = torch.as_tensor(mel_basis, dtype=torch.float32).to(device).contiguous()

    def __call__(self, low, y=None, workspace=None, stream=None):
        C, T = low.shape
        sp = self.spec
        y = torch.empty((C, sp.ratio * T), device=low.device, dtype=torch.float32) \
            if y is None else y
        if workspace is None:
            need = int(lib().bv_bwe_tail_workspace_size(ctypes.byref(self.dec.cfg), C, T,
                                                         sp.n_fft, sp.hop, sp.n_mels, sp.ratio))
            if need == 0:
                raise BVError(2, last_error())
            workspace = torch.empty(need // 4 + 64, device=low.device, dtype=torch.float32)
        _check(lib().bv_bwe_tail(ctypes.byref(self.dec.cfg), ctypes.byref(self.dec.weights),
                                 _ptr(low), C, T, _ptr(self.basis), sp.n_fft, sp.hop,
                                 _ptr(self.mel_basis), sp.n_mels, sp.ratio, _ptr(y),
                                 _ptr(workspace), workspace.numel() * 4, _stream(stream)))
        return y
