"""The C ABI without a GPU: the library loads, exports every declared symbol,
designs the filter on the host, and rejects bad arguments before touching a
device.  Valid compute calls on a machine without a GPU must fail with
BV_ERR_CUDA -- there is no CPU fallback."""
import ctypes
import os
import re

import numpy as np
import pytest

from bigvgan_waveform_decoder_alias_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bv.h")


@pytest.fixture(scope="module")
def nat():
    from bigvgan_waveform_decoder_alias_b200 import build_native, native
    build_native.build()
    native.lib()
    return native


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(bv_[a-z0-9_]+)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(nat):
    names = declared_functions()
    assert len(names) >= 15, names
    L = nat.lib()
    for n in names:
        assert hasattr(L, n), f"libbv.so does not export {n}"


def test_version(nat):
    assert "sm_100a" in nat.version()


def test_filter_design_matches_oracle(nat, oracle):
    got = nat.bv_filter_design(0.25, 0.3, 12)
    want = oracle.kaiser_sinc(0.25, 0.3, 12)
    np.testing.assert_array_equal(got, want)
    for k, c, hw in ((8, 0.25, 0.3), (16, 0.2, 0.25), (11, 0.25, 0.3), (24, 0.25, 0.1)):
        np.testing.assert_array_equal(nat.bv_filter_design(c, hw, k),
                                      oracle.kaiser_sinc(c, hw, k))


def test_filter_design_rejects_bad_arguments(nat):
    L = nat.lib()
    buf = (ctypes.c_float * 12)()
    assert L.bv_filter_design(0.25, 0.3, 0, buf) == 1
    assert L.bv_filter_design(0.25, 0.3, 65, buf) == 1
    assert L.bv_filter_design(0.0, 0.3, 12, buf) == 1
    assert L.bv_filter_design(0.25, -1.0, 12, buf) == 1
    assert L.bv_filter_design(0.25, 0.3, 12, None) == 1


FAKE = ctypes.c_void_p(0x10000)   # never dereferenced: the calls fail first
FAKE2 = ctypes.c_void_p(0x90000000)


def test_activation_argument_errors(nat):
    L = nat.lib()
    s = ctypes.c_void_p(0)
    assert L.bv_activation1d(None, FAKE2, 1, 1, 8, FAKE, FAKE, FAKE, FAKE, 1e-9, s) == 1
    assert L.bv_activation1d(FAKE, FAKE2, 0, 1, 8, FAKE, FAKE, FAKE, FAKE, 1e-9, s) == 2
    assert L.bv_activation1d(FAKE, FAKE, 1, 1, 8, FAKE, FAKE, FAKE, FAKE, 1e-9, s) == 1  # overlap
    assert "overlap" in nat.last_error()
    assert L.bv_activation1d(ctypes.c_void_p(0x10002), FAKE2, 1, 1, 8, FAKE, FAKE, FAKE, FAKE,
                             1e-9, s) == 1  # misaligned


def test_conv_argument_errors(nat):
    L = nat.lib()
    s = ctypes.c_void_p(0)
    ep = nat.Epilogue(None, 1.0, 0, 0)
    # output length < 1
    assert L.bv_conv1d(FAKE, 1, 4, 3, FAKE, None, 4, 11, 5, 0, ctypes.byref(ep), FAKE2, s) == 2
    assert L.bv_conv1d(FAKE, 1, 4, 30, FAKE, None, 4, 33, 1, 16, ctypes.byref(ep), FAKE2, s) == 2
    ep.final_act = 7
    assert L.bv_conv1d(FAKE, 1, 4, 30, FAKE, None, 4, 3, 1, 1, ctypes.byref(ep), FAKE2, s) == 1
    assert L.bv_conv_transpose1d(FAKE, 1, 4, 8, FAKE, None, 4, 10, 17, 0, FAKE2, s) == 2
    assert L.bv_conv_transpose1d(None, 1, 4, 8, FAKE, None, 4, 10, 5, 2, FAKE2, s) == 1


def test_no_cpu_fallback(nat):
    """A valid request with no usable GPU returns BV_ERR_CUDA."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    L = nat.lib()
    s = ctypes.c_void_p(0)
    rc = L.bv_activation1d(FAKE, FAKE2, 1, 1, 8, FAKE, FAKE, FAKE, FAKE, 1e-9, s)
    assert rc == 4, nat.last_error()
    ep = nat.Epilogue(None, 1.0, 0, 0)
    assert L.bv_conv1d(FAKE, 1, 4, 30, FAKE, None, 4, 3, 1, 1, ctypes.byref(ep), FAKE2, s) == 4


def test_decoder_bookkeeping(nat, oracle):
    for geo in (synth.H3, synth.LTX, synth.tiny_geometry()):
        cfg = nat.decoder_config(geo)
        assert nat.bv_decoder_param_count(cfg) == synth.param_count(geo) == oracle.param_count(geo)
        L = nat.lib()
        assert L.bv_decoder_output_length(ctypes.byref(cfg), 400) == 400 * geo.hop
        assert L.bv_decode_workspace_size(ctypes.byref(cfg), 2, 400) > 0
    cfg = nat.decoder_config(synth.H3)
    cfg.block_kernel[0] = 4  # even kernels break "same" padding
    assert nat.bv_decoder_param_count(cfg) == -1


def test_conv_split_flag_is_checked_and_changes_no_sizes(nat):
    """tf32_only is 0 or 1; the split it selects fits the same buffers (an
    fp16 split row of 64-channel blocks takes at most the bytes of a tf32 one
    of 32-channel blocks), so no workspace or prepared size depends on it."""
    L = nat.lib()
    for geo in (synth.H3, synth.LTX):
        a = nat.decoder_config(geo, 200, 16)
        b = nat.decoder_config(geo, 200, 16, tf32_only=True)
        assert b.tf32_only == 1 and a.tf32_only == 0
        for f in (L.bv_decode_workspace_size, L.bv_decode_workspace_size_prepared):
            assert f(ctypes.byref(a), 2, 2400) == f(ctypes.byref(b), 2, 2400) > 0
        assert L.bv_decoder_prepared_size(ctypes.byref(a)) == \
            L.bv_decoder_prepared_size(ctypes.byref(b)) > 0
    bad = nat.decoder_config(synth.H3)
    bad.tf32_only = 2
    assert L.bv_decode_workspace_size(ctypes.byref(bad), 2, 400) == 0
    assert "tf32_only" in nat.last_error()


def test_decode_workspace_grows_with_tiles(nat):
    L = nat.lib()
    untiled = nat.decoder_config(synth.H3)
    tiled = nat.decoder_config(synth.H3, 200, 16)
    a = L.bv_decode_workspace_size(ctypes.byref(untiled), 2, 400)
    b = L.bv_decode_workspace_size(ctypes.byref(tiled), 2, 400)
    c = L.bv_decode_workspace_size(ctypes.byref(tiled), 2, 2400)
    assert a > 0 and b > 0 and c > b
    # 400 frames = 2 full tiles + a last one of 32 frames
    assert L.bv_decode_workspace_size(ctypes.byref(tiled), 2, 200) == \
        L.bv_decode_workspace_size(ctypes.byref(untiled), 2, 200)


def test_decode_rejects_small_workspace(nat):
    L = nat.lib()
    geo = synth.tiny_geometry()
    cfg = nat.decoder_config(geo)
    w = nat.DecoderWeights()
    flat = ctypes.c_void_p(0x100000)
    assert L.bv_decoder_weights_from_flat(ctypes.byref(cfg), flat, FAKE, FAKE, ctypes.byref(w)) == 0
    need = L.bv_decode_workspace_size(ctypes.byref(cfg), 2, 6)
    rc = L.bv_decode(ctypes.byref(cfg), ctypes.byref(w), ctypes.c_void_p(0x200000), 2, 6,
                     ctypes.c_void_p(0x300000), ctypes.c_void_p(0x40000000), need - 1,
                     ctypes.c_void_p(0))
    assert rc == 3
    # weights whose block kernel disagrees with the config
    w.amp[0][1].kernel_size = 5
    rc = L.bv_decode(ctypes.byref(cfg), ctypes.byref(w), ctypes.c_void_p(0x200000), 2, 6,
                     ctypes.c_void_p(0x300000), ctypes.c_void_p(0x40000000), need,
                     ctypes.c_void_p(0))
    assert rc == 1


def test_weights_from_flat_walks_module_order(nat):
    geo = synth.tiny_geometry()
    cfg = nat.decoder_config(geo)
    w = nat.DecoderWeights()
    base = 0x100000
    nat.lib().bv_decoder_weights_from_flat(ctypes.byref(cfg), ctypes.c_void_p(base), FAKE,
                                           FAKE, ctypes.byref(w))
    off, offs = 0, {}
    for name, shape, _ in synth.param_layout(geo):
        offs[name] = base + 4 * off
        off += int(np.prod(shape))
    assert w.pre_w == offs["conv_pre.w"] and w.pre_b == offs["conv_pre.b"]
    assert w.up_w[2] == offs["ups.2.w"]
    a = w.amp[1][2]
    assert a.conv1_w[1] == offs["stage1.block2.unit1.conv1.w"]
    assert a.act_log_beta[3] == offs["stage1.block2.unit1.act2.log_beta"]
    assert w.post_w == offs["conv_post.w"] and w.post_b == offs["conv_post.b"]
