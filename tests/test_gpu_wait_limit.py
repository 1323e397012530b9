"""The bounded waits of the tensor-core kernels, made to run out.

Every mbarrier wait in the tcgen05 kernels polls a bounded number of times
(2^26 by default) before it gives up; the CTA (and its pair) then stops
issuing work, lets the copies and MMAs it issued finish, frees its tensor
memory and reports the failure in the status word that bv_sync_status
reads.  Here the library's testing hook lowers the limit to 0 polls, so the
first wait of a launch that is not already satisfied gives up: both
tensor-core kernels (the time-major CTA-pair conv behind bv_act_conv1d and
the [B, C, T] conv behind bv_conv1d) must report BV_ERR_TIMEOUT and leave
the context usable -- the same calls at the default limit then match the
oracle.  Nothing is planted: the kernels and their inputs are the normal
ones, only the patience of their waits changes.
"""
import numpy as np
import pytest
import torch

from bigvgan_waveform_decoder_alias_b200 import synth

pytestmark = pytest.mark.gpu

LAYER_TOL = 1e-5
BV_ERR_TIMEOUT = 5


def rel_l2(got, want):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    return float(np.linalg.norm(got - want) / np.linalg.norm(want))


@pytest.fixture(scope="module")
def nat():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bigvgan_waveform_decoder_alias_b200 import build_native, native
    build_native.build()
    native.lib()
    return native


def _status(nat):
    import ctypes
    return nat.lib().bv_sync_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_wait_limit_zero_reports_timeout_and_context_survives(nat, oracle):
    s = synth.NormalStream(321)
    C, T, K, d = 128, 1000, 7, 3
    x = s.normal((2, C, T))
    la, lb = s.normal((C,), 0.0, 0.1), s.normal((C,), 0.0, 0.1)
    w = s.normal((C, C, K), 0.0, 0.02)
    b = s.normal((C,), 0.0, 0.02)
    filt = torch.from_numpy(nat.bv_filter_design()).cuda()
    xd, lad, lbd = (torch.from_numpy(a).cuda() for a in (x, la, lb))
    wd, bd = torch.from_numpy(w).cuda(), torch.from_numpy(b).cuda()
    pad = (K * d - d) // 2

    def act_conv():
        return nat.bv_act_conv1d(xd, lad, lbd, filt, wd, bd, d, pad)

    def conv():  # [B, C, T] tensor-core kernel (K2')
        return nat.bv_conv1d(xd, wd, bd, d, pad)

    nat.timing(True)
    nat.timing_reset()
    try:
        act_conv()
        conv()
        torch.cuda.synchronize()
        classes = nat.timing_read()
    finally:
        nat.timing(False)
        nat.timing_reset()
    assert "conv1d_tm_f16" in classes and "conv1d_tc" in classes, classes
    assert _status(nat) == 0

    prev = nat.set_wait_limit(0)
    try:
        act_conv()
        st_tm = _status(nat)
        conv()
        st_tc = _status(nat)
    finally:
        nat.set_wait_limit(-1)
    assert prev == 1 << 26
    assert st_tm == BV_ERR_TIMEOUT, st_tm
    assert st_tc == BV_ERR_TIMEOUT, st_tc
    assert "gave up" in nat.last_error()

    # the default limit is back, the context still works and the status is clean
    assert nat.set_wait_limit(-1) == 1 << 26
    h = oracle.activation1d(x, la, lb)
    y1 = act_conv().cpu().numpy()
    assert rel_l2(y1, oracle.conv1d(h, w, b, d, pad)) < LAYER_TOL
    y2 = conv().cpu().numpy()
    assert rel_l2(y2, oracle.conv1d(x, w, b, d, pad)) < LAYER_TOL
    assert _status(nat) == 0


BV_ERR_RANGE = 7


def test_fp16_operand_range_is_reported(nat, oracle):
    """The fp16 time-major path (64 channels) on activations past fp16's range
    (inputs of order 1e5; the activation is about its input there): the status
    word reports BV_ERR_RANGE, and the next call on ordinary inputs is clean and
    matches the oracle."""
    s = synth.NormalStream(322)
    C, T, K, d = 64, 300, 3, 1
    x = s.normal((2, C, T))
    la, lb = s.normal((C,), 0.0, 0.1), s.normal((C,), 0.0, 0.1)
    w = s.normal((C, C, K), 0.0, 0.02)
    b = s.normal((C,), 0.0, 0.02)
    filt = torch.from_numpy(nat.bv_filter_design()).cuda()
    lad, lbd = (torch.from_numpy(a).cuda() for a in (la, lb))
    wd, bd = torch.from_numpy(w).cuda(), torch.from_numpy(b).cuda()
    assert _status(nat) == 0
    big = torch.from_numpy(1.0e5 * x).cuda()
    nat.bv_act_conv1d(big, lad, lbd, filt, wd, bd, d, 1)
    assert _status(nat) == BV_ERR_RANGE
    assert "fp16" in nat.last_error()
    y = nat.bv_act_conv1d(torch.from_numpy(x).cuda(), lad, lbd, filt, wd, bd, d, 1)
    assert _status(nat) == 0
    want = oracle.conv1d(oracle.activation1d(x, la, lb), w, b, d, 1)
    assert rel_l2(y.cpu().numpy(), want) < LAYER_TOL


def test_fp16_operand_range_is_reported_for_transposed_convs(nat, oracle):
    """The transposed conv's fp16 planes (64 input channels) from inputs of
    order 1e5: BV_ERR_RANGE; then ordinary inputs are clean and match."""
    s = synth.NormalStream(323)
    Cin, Cout, S, T = 64, 48, 2, 300
    K, pad = 2 * S, S // 2
    x = s.normal((2, Cin, T))
    w = s.normal((Cin, Cout, K), 0.0, 0.02)
    b = s.normal((Cout,), 0.0, 0.02)
    wd, bd = torch.from_numpy(w).cuda(), torch.from_numpy(b).cuda()
    assert _status(nat) == 0
    nat.bv_conv_transpose1d_ws(torch.from_numpy(1.0e5 * x).cuda(), wd, bd, S, pad)
    assert _status(nat) == BV_ERR_RANGE
    y = nat.bv_conv_transpose1d_ws(torch.from_numpy(x).cuda(), wd, bd, S, pad)
    assert _status(nat) == 0
    assert rel_l2(y.cpu().numpy(), oracle.conv_transpose1d(x, w, b, S, pad)) < LAYER_TOL


def test_fp16_weight_range_is_reported(nat, oracle):
    """Weights of 16 or more leave fp16's range once scaled by 2^12 for the
    fp16 split: the split reports BV_ERR_RANGE instead of infinities."""
    s = synth.NormalStream(324)
    C, T, K, d = 64, 200, 3, 1
    x = s.normal((2, C, T))
    la, lb = s.normal((C,), 0.0, 0.1), s.normal((C,), 0.0, 0.1)
    w = s.normal((C, C, K), 0.0, 0.02)
    w[3, 5, 1] = 20.0
    b = s.normal((C,), 0.0, 0.02)
    filt = torch.from_numpy(nat.bv_filter_design()).cuda()
    lad, lbd = (torch.from_numpy(a).cuda() for a in (la, lb))
    assert _status(nat) == 0
    nat.bv_act_conv1d(torch.from_numpy(x).cuda(), lad, lbd, filt, torch.from_numpy(w).cuda(),
                      torch.from_numpy(b).cuda(), d, 1)
    assert _status(nat) == BV_ERR_RANGE
