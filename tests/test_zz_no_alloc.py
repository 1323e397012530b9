"""bv_amp_block_static: the AMP block whose scratch is a static device array
inside the library, for callers that cannot allocate device memory while
they decode (real-time audio threads, hosts with a fixed memory budget).

Called through the C ABI and checked against bv_amp_block (the same block
with a caller workspace) on two calls in a row, so the second call runs on
scratch the first one left behind.  This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from bigvgan_waveform_decoder_alias_b200 import synth

pytestmark = pytest.mark.gpu

LAYER_TOL = 1e-5  # the tolerance of the layer parity tests


def rel_l2(got, want):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    return float(np.linalg.norm(got - want) / np.linalg.norm(want))


def test_static_scratch_amp_block_matches_workspace_version():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bigvgan_waveform_decoder_alias_b200 import build_native, native
    build_native.build()
    L = native.lib()
    torch.cuda.set_device(0)
    filt = torch.from_numpy(native.bv_filter_design(0.25, 0.3, 12)).cuda()

    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = [synth.AMP_BLOCK_C32, synth.AmpWorkload("c96", 2, 96, 3001, 7, (1, 3, 5), seed=5)]
    params = {}
    for w in cases:
        x, flat = w.make()
        tensors, off = {}, 0
        for name, shape, _ in w.layout():
            n = int(np.prod(shape))
            tensors[name] = torch.from_numpy(flat[off:off + n].reshape(shape)).cuda()
            off += n
        p = native.amp_params(w.kernel, w.dilations, tensors, filt)
        params[w.name] = (p, tensors)  # the tensors must outlive the pointers in p
        xd = torch.from_numpy(x).cuda()
        want = native.bv_amp_block(xd, p).cpu().numpy()
        for call in range(2):
            y = torch.full_like(xd, float("nan"))
            rc = L.bv_amp_block_static(ctypes.c_void_p(xd.data_ptr()), w.batch, w.channels,
                                       w.length, ctypes.byref(p), ctypes.c_void_p(y.data_ptr()),
                                       1.0, 0, stream)
            assert rc == 0, native.last_error()
            got = y.cpu().numpy()
            assert np.isfinite(got).all(), (w.name, call)
            assert rel_l2(got, want) < LAYER_TOL, (w.name, call)

        # scale and accumulate behave as in bv_amp_block
        y0 = torch.from_numpy(synth.NormalStream(3).normal(x.shape)).cuda()
        y = y0.clone()
        rc = L.bv_amp_block_static(ctypes.c_void_p(xd.data_ptr()), w.batch, w.channels,
                                   w.length, ctypes.byref(p), ctypes.c_void_p(y.data_ptr()),
                                   0.5, 1, stream)
        assert rc == 0, native.last_error()
        ref = 0.5 * want.astype(np.float64) + y0.cpu().numpy()
        assert rel_l2(y.cpu().numpy(), ref) < LAYER_TOL

    # the 32-channel block's own parameters for the size limits
    p32, _ = params[synth.AMP_BLOCK_C32.name]
    limit = 1 << 20  # BV_AMP_STATIC_MAX_ELEMS in include/bv.h
    # exactly the limit: B * C * T == BV_AMP_STATIC_MAX_ELEMS runs and matches
    t_max = limit // 32
    xd = torch.from_numpy(synth.NormalStream(4).normal((1, 32, t_max))).cuda()
    want = native.bv_amp_block(xd, p32).cpu().numpy()
    y = torch.full_like(xd, float("nan"))
    rc = L.bv_amp_block_static(ctypes.c_void_p(xd.data_ptr()), 1, 32, t_max, ctypes.byref(p32),
                               ctypes.c_void_p(y.data_ptr()), 1.0, 0, stream)
    assert rc == 0, native.last_error()
    assert rel_l2(y.cpu().numpy(), want) < LAYER_TOL

    # one element more than the static scratch holds: a clear error, output untouched
    big_t = t_max + 1
    xd = torch.zeros((1, 32, big_t), device="cuda")
    y = torch.full_like(xd, 7.0)
    rc = L.bv_amp_block_static(ctypes.c_void_p(xd.data_ptr()), 1, 32, big_t, ctypes.byref(p32),
                               ctypes.c_void_p(y.data_ptr()), 1.0, 0, stream)
    assert rc == 3 and "static scratch limit" in native.last_error()
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())
