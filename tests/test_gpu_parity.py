"""Parity of the CUDA path (through the C ABI) with the oracle, element by
element on the same seeded inputs.

Tolerances (the decoder's accuracy target): a single layer within 1e-5
relative L2 of the oracle given the same float input, the whole waveform
within 1e-4.  Spot checks of full-size tensors compare sampled outputs that
the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

from bigvgan_waveform_decoder_alias_b200 import synth

pytestmark = pytest.mark.gpu

LAYER_TOL = 1e-5
WAVE_TOL = 1e-4


def rel_l2(got, want):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


@pytest.fixture(scope="module")
def nat():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bigvgan_waveform_decoder_alias_b200 import build_native, native
    build_native.build()
    native.lib()
    return native


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.detach().cpu().numpy()


@pytest.fixture(scope="module")
def filt(oracle, nat):
    f = nat.bv_filter_design(0.25, 0.3, 12)
    np.testing.assert_array_equal(f, oracle.kaiser_sinc())
    return dev(f)


# -------------------------------------------------------------- activation

ACT_SHAPES = [(1, 1, 1), (1, 1, 2), (1, 3, 3), (2, 1, 5), (1, 2, 13), (1, 1, 1023),
              (2, 3, 1024), (1, 2, 1025), (2, 2, 2049), (1, 5, 5000), (3, 4, 4100)]


@pytest.mark.parametrize("B,C,T", ACT_SHAPES)
def test_activation_matches_oracle(nat, oracle, filt, B, C, T):
    s = synth.NormalStream(1000 + 7 * T + C)
    x = s.normal((B, C, T), 0.0, 2.0)
    la, lb = s.normal((C,), 0.0, 0.3), s.normal((C,), 0.0, 0.3)
    y = host(nat.bv_activation1d(dev(x), dev(la), dev(lb), filt))
    want = oracle.activation1d(x, la, lb)
    assert y.shape == want.shape
    assert rel_l2(y, want) < LAYER_TOL
    np.testing.assert_allclose(y, want, rtol=1e-5, atol=1e-5)


def test_activation_large_arguments(nat, oracle, filt):
    """Rows whose SnakeBeta argument e^alpha u passes sin^2's fast-path limit
    (|a u| > 51472, where the kernel takes the scalar sin^2 per pair) while
    |x| stays near 1, so the SnakeBeta term is as large as the signal itself;
    the other rows stay on the fast path.

    sin^2 of a large float argument is ill-conditioned: a = expf(log_alpha)
    carries up to 2 ulp, the fast path's a/pi two more roundings, u up to 6
    roundings of its taps' products and the product one more, so the
    argument is known to about |a u| 1e-6 (bounded with the window's largest
    |x|), and
    sin^2 moves by at most that much (|d sin^2 z / dz| <= 1); the scalar sin^2
    itself is within 5e-6.  Through 1/(e^beta + eps) and the 12 down-sampling
    taps that bounds each output's error; the test checks every element
    against that bound (plus the float rounding of the rest), and the
    fast-path rows at the layer tolerance."""
    s = synth.NormalStream(99)
    B, C, T = 2, 6, 5000
    x = s.normal((B, C, T))
    big = np.arange(C) % 2 == 0
    la = np.where(big, np.log(9.0e4), 0.0) + s.normal((C,), 0.0, 0.1)
    la = la.astype(np.float32)
    lb = s.normal((C,), 0.0, 0.1)
    y = host(nat.bv_activation1d(dev(x), dev(la), dev(lb), filt)).astype(np.float64)
    want = oracle.activation1d(x, la, lb, store_f64=True).astype(np.float64)
    assert np.isfinite(y).all()
    f = oracle.kaiser_sinc().astype(np.float64)
    up_abs = max(np.abs(2 * f[1::2]).sum(), np.abs(2 * f[0::2]).sum())
    # largest |x| each output's 2x-rate inputs reach (x[t - 8 .. t + 8])
    ax = np.abs(x.astype(np.float64))
    pad = np.pad(ax, ((0, 0), (0, 0), (8, 8)), mode="edge")
    xmax = np.max(np.stack([pad[..., k:k + T] for k in range(17)]), axis=0)
    a = np.exp(la.astype(np.float64))[None, :, None]
    ib = 1.0 / (np.exp(lb.astype(np.float64)) + 1e-9)[None, :, None]
    zmax = a * up_abs * xmax
    assert (zmax[:, big] > 51472).mean() > 0.9  # the big rows do take the scalar sin^2
    bound = np.abs(f).sum() * (ib * (zmax * 1e-6 + 5e-6)) + 2e-6 * (np.abs(want) + 1)
    err = np.abs(y - want)
    assert (err <= bound).all(), float((err / bound).max())
    # the quiet rows: the ordinary layer tolerance
    assert rel_l2(y[:, ~big], want[:, ~big]) < LAYER_TOL
    # the SnakeBeta term is a large part of the big rows' output
    ident = oracle.activation1d(x, la, np.full(C, 80.0, np.float32), store_f64=True)
    snake = want[:, big] - ident[:, big]
    assert np.linalg.norm(snake) > 0.3 * np.linalg.norm(want[:, big])
    # and, over the whole of it, the error is the small fraction of that term
    # the argument's float rounding predicts (about 1 %), not a wrong constant
    assert np.linalg.norm(y[:, big] - want[:, big]) < 0.05 * np.linalg.norm(snake)


def test_activation_constant_rows_exact_form(nat, filt):
    """Constant rows map to c + sin^2(e^a c)/(e^b + eps) everywhere, edges too."""
    C, T = 4, 3000
    cs = np.array([0.3, -1.7, 2.5, np.pi / 2], np.float32)
    la = np.array([0.05, -0.2, 0.1, 0.0], np.float32)
    lb = np.array([-0.1, 0.15, 0.0, 0.0], np.float32)
    x = np.repeat(cs[None, :, None], T, axis=2)
    y = host(nat.bv_activation1d(dev(x), dev(la), dev(lb), filt))
    for c in range(C):
        want = cs[c] + np.sin(np.exp(la[c]) * cs[c]) ** 2 / (np.exp(lb[c]) + 1e-9)
        np.testing.assert_allclose(y[0, c], want, rtol=2e-6, atol=2e-6)


def test_sin_squared_accuracy(nat):
    """The kernel's own sin^2 (Cody-Waite reduction by pi, Taylor series of
    sin to r^13) against double precision, and against CUDA's sinf squared."""
    rng = np.random.default_rng(0)
    z = np.concatenate([np.linspace(-8, 8, 20001), rng.normal(0, 30, 200000),
                        rng.uniform(-65536, 65536, 200000),
                        np.array([0.0, np.pi / 2, np.pi, 1e-30, -1e-30, 65536.0, 65537.0,
                                  1e5, -3e6, 1e30])]).astype(np.float32)
    zd = dev(z)
    got = host(nat.bv_sin_squared(zd)).astype(np.float64)
    exact = np.sin(z.astype(np.float64)) ** 2
    # the argument is exact (a float); the error is the reduction and series
    err = np.abs(got - exact)
    small = np.abs(z) <= 1024
    assert err[small].max() < 4e-7, err[small].max()
    assert err.max() < 4e-6, err.max()
    cuda_sinf2 = host(torch.sin(zd)).astype(np.float64) ** 2
    assert np.abs(got - cuda_sinf2)[small].max() < 5e-7


def test_activation_full_size_sweep_point(nat, oracle, filt):
    """The activation workload at full size [2, 512, 65536], every element."""
    w = synth.ACT_SWEEP
    x, la, lb = w.make()
    y = host(nat.bv_activation1d(dev(x), dev(la), dev(lb), filt))
    want = oracle.activation1d(x, la, lb)
    assert rel_l2(y, want) < LAYER_TOL
    assert np.abs(y - want).max() < 1e-4


@pytest.mark.parametrize("B,C,T", [(1, 8, 128 * 1200 + 1), (1, 7, 128 * 1500 + 2),
                                   (2, 3, 128 * 900 + 130)])
def test_activation_multi_tile_ranges_and_short_last_tiles(nat, oracle, filt, B, C, T):
    """Enough tiles that warps own several consecutive 128-output tiles (so a
    tile's down-sampling reads the next tile's first 2x-rate values), rows
    whose last tile holds 1, 2 or 2 + 128 outputs (the replicate padding then
    reaches into the previous tile's reads), and odd row counts; every
    element against the oracle."""
    s = synth.NormalStream(5000 + C + T)
    x = s.normal((B, C, T), 0.0, 1.5)
    la, lb = s.normal((C,), 0.0, 0.3), s.normal((C,), 0.0, 0.3)
    y = host(nat.bv_activation1d(dev(x), dev(la), dev(lb), filt))
    want = oracle.activation1d(x, la, lb)
    assert rel_l2(y, want) < LAYER_TOL
    tail = slice(T - 300, T)
    assert rel_l2(y[..., tail], want[..., tail]) < LAYER_TOL
    assert np.abs(y - want).max() < 1e-4


@pytest.mark.parametrize("C,T", [(64, 262144), (1536, 4096), (768, 16384)])
def test_activation_sweep_shapes_sampled(nat, oracle, filt, C, T):
    s = synth.NormalStream(C + T)
    x = s.normal((2, C, T))
    la, lb = s.normal((C,), 0.0, 0.1), s.normal((C,), 0.0, 0.1)
    y = host(nat.bv_activation1d(dev(x), dev(la), dev(lb), filt))
    rng = np.random.default_rng(C + T)
    pts = np.stack([rng.integers(0, 2, 3000), rng.integers(0, C, 3000),
                    rng.integers(0, T, 3000)], 1)
    pts = np.concatenate([pts, [[0, 0, 0], [1, C - 1, T - 1], [0, 1, T - 2]]])
    want = oracle.activation1d_points(x, la, lb, pts)
    got = y[pts[:, 0], pts[:, 1], pts[:, 2]]
    assert rel_l2(got, want) < LAYER_TOL


# ------------------------------------------------------------------- convs

CONV_CASES = [(C, K, d, T) for (C, T) in ((12, 1000), (32, 333), (48, 257), (96, 130), (128, 300))
              for K in (3, 7, 11) for d in (1, 3, 5)]


@pytest.mark.parametrize("C,K,d,T", CONV_CASES)
def test_conv1d_matches_oracle(nat, oracle, C, K, d, T):
    s = synth.NormalStream(3000 + C * 7 + K * 3 + d + T)
    B = 2
    x = s.normal((B, C, T))
    w = s.normal((C, C, K), 0.0, 0.02)
    b = s.normal((C,), 0.0, 0.02)
    pad = (K * d - d) // 2
    y = host(nat.bv_conv1d(dev(x), dev(w), dev(b), d, pad))
    want = oracle.conv1d(x, w, b, d, pad)
    assert rel_l2(y, want) < LAYER_TOL


@pytest.mark.parametrize("Cin,Cout,K,T", [(32, 1536, 7, 400), (64, 1024, 7, 500),
                                          (12, 1, 7, 5001), (16, 1, 7, 777), (3, 5, 1, 9),
                                          (7, 9, 5, 1), (1, 1, 3, 2), (200, 130, 3, 65)])
def test_conv1d_channel_changes(nat, oracle, Cin, Cout, K, T):
    s = synth.NormalStream(Cin * 1000 + Cout + K + T)
    x = s.normal((2, Cin, T))
    w = s.normal((Cout, Cin, K), 0.0, 0.05)
    b = s.normal((Cout,), 0.0, 0.05)
    y = host(nat.bv_conv1d(dev(x), dev(w), dev(b), 1, (K - 1) // 2))
    assert rel_l2(y, oracle.conv1d(x, w, b, 1, (K - 1) // 2)) < LAYER_TOL


def test_conv1d_unpadded_no_bias(nat, oracle):
    s = synth.NormalStream(17)
    x = s.normal((1, 20, 100))
    w = s.normal((30, 20, 5), 0.0, 0.1)
    y = host(nat.bv_conv1d(dev(x), dev(w), None, 3, 0))
    want = oracle.conv1d(x, w, None, 3, 0)
    assert y.shape == (1, 30, 88) and rel_l2(y, want) < LAYER_TOL


@pytest.mark.parametrize("C", [48, 24, 13])
@pytest.mark.parametrize("final_act", [0, 1, 2])
def test_conv1d_epilogue(nat, oracle, final_act, C):
    """y = final(scale * (conv + bias + residual) + y_old), on the tensor-core
    path (48 channels) and the narrow FP32 kernel (24; 13 with an odd row
    pitch and a partial channel group)."""
    s = synth.NormalStream(50 + final_act + C)
    T = 700 + C % 2
    x = s.normal((2, C, T))
    w = s.normal((C, C, 7), 0.0, 0.1)
    b = s.normal((C,), 0.0, 0.1)
    r = s.normal((2, C, T))
    y0 = s.normal((2, C, T))
    yd = dev(y0)
    nat.bv_conv1d(dev(x), dev(w), dev(b), 3, 9, residual=dev(r), scale=1.0 / 3.0,
                  accumulate=True, final_act=final_act, y=yd)
    got = host(yd).astype(np.float64)
    conv = oracle.conv1d(x, w, b, 3, 9, store_f64=True).astype(np.float64)
    want = (conv + r) * (1.0 / 3.0) + y0
    if final_act == 1:
        want = np.clip(want, -1, 1)
    elif final_act == 2:
        want = np.tanh(want)
    assert rel_l2(got, want) < LAYER_TOL


@pytest.mark.parametrize("C", [96, 24])
def test_conv1d_inplace_residual(nat, oracle, C):
    s = synth.NormalStream(77 + C)
    T = 513
    x = s.normal((1, C, T))
    w = s.normal((C, C, 3), 0.0, 0.05)
    cur = s.normal((1, C, T))
    cd = dev(cur)
    nat.bv_conv1d(dev(x), dev(w), None, 5, 5, residual=cd, y=cd)
    want = oracle.conv1d(x, w, None, 5, 5, store_f64=True).astype(np.float64) + cur
    assert rel_l2(host(cd), want) < LAYER_TOL


@pytest.mark.parametrize("S,T,Cin,Cout", [(5, 400, 64, 48), (5, 1, 16, 8), (2, 2001, 48, 24),
                                          (2, 3, 12, 12), (3, 50, 20, 10), (4, 77, 24, 40),
                                          (6, 33, 16, 16), (8, 20, 8, 12)])
def test_conv_transpose1d_matches_oracle(nat, oracle, S, T, Cin, Cout):
    s = synth.NormalStream(4000 + S * 100 + T)
    K = 2 * S
    pad = (K - S) // 2
    x = s.normal((2, Cin, T))
    w = s.normal((Cin, Cout, K), 0.0, 0.05)
    b = s.normal((Cout,), 0.0, 0.05)
    y = host(nat.bv_conv_transpose1d(dev(x), dev(w), dev(b), S, pad))
    want = oracle.conv_transpose1d(x, w, b, S, pad)
    assert y.shape == want.shape
    assert rel_l2(y, want) < LAYER_TOL


@pytest.mark.parametrize("Cin,Cout,S,K,pad,T", [(48, 24, 2, 4, 1, 5001), (24, 12, 2, 4, 1, 1),
                                                (64, 32, 2, 4, 1, 777), (17, 5, 2, 3, 0, 130),
                                                (8, 1, 1, 3, 1, 600), (33, 20, 2, 8, 3, 513),
                                                (40, 32, 1, 4, 0, 1025), (12, 12, 2, 4, 1, 1024)])
def test_conv_transpose1d_narrow_kernel(nat, oracle, Cin, Cout, S, K, pad, T):
    """The narrow polyphase ConvT (at most 64 in, 32 out channels, strides 1
    and 2): odd and even kernels, several staged channel chunks, a padded
    output-channel group, ragged and one-sample inputs; every output."""
    s = synth.NormalStream(19000 + Cin + Cout + K + T)
    x = s.normal((2, Cin, T))
    w = s.normal((Cin, Cout, K), 0.0, 0.1)
    b = s.normal((Cout,), 0.0, 0.1)
    y = host(nat.bv_conv_transpose1d(dev(x), dev(w), dev(b), S, pad))
    want = oracle.conv_transpose1d(x, w, b, S, pad)
    assert y.shape == want.shape
    assert rel_l2(y, want) < LAYER_TOL
    np.testing.assert_allclose(y, want, rtol=1e-4, atol=1e-5)


def test_conv_transpose1d_general_kernel(nat, oracle):
    s = synth.NormalStream(99)
    x = s.normal((1, 10, 37))
    for S, K, pad in ((5, 11, 3), (2, 3, 0), (4, 4, 0), (3, 9, 4)):
        w = s.normal((10, 6, K), 0.0, 0.1)
        y = host(nat.bv_conv_transpose1d(dev(x), dev(w), None, S, pad))
        assert rel_l2(y, oracle.conv_transpose1d(x, w, None, S, pad)) < LAYER_TOL


# Shapes that take the tensor-core path (tcgen05, 3xTF32): partial output
# tiles (Cout not a multiple of 128), partial k chunks (Cin K not a multiple
# of 32), partial input-channel blocks, short and ragged time axes, the
# largest halo, and every epilogue.
TC_CASES = [(64, 64, 3, 1, 200), (128, 128, 3, 1, 1), (128, 128, 7, 3, 5), (96, 96, 11, 5, 130),
            (192, 192, 11, 5, 257), (64, 128, 3, 1, 129), (40, 200, 7, 1, 300),
            (384, 384, 11, 5, 127), (768, 768, 3, 1, 400), (32, 1536, 7, 1, 77),
            (256, 256, 7, 3, 1024), (100, 300, 11, 1, 513), (48, 48, 7, 3, 700),
            (48, 48, 11, 5, 77), (64, 40, 3, 1, 300), (96, 112, 7, 1, 130), (80, 80, 3, 1, 9)]


# The time-major conv's timer classes: 3xTF32, and the fp16 split that convs
# fed by the time-major activation take for channel counts that are
# multiples of 8 from 48 up.
TM_CLASSES = ("conv1d_tm", "conv1d_tm_f16")
TMT_CLASSES = ("conv_transpose1d_tm", "conv_transpose1d_tm_f16")


def _has_tm(classes):
    return any(c in classes for c in TM_CLASSES)


def _has_tmt(classes):
    return any(c in classes for c in TMT_CLASSES)


def _kernel_classes(nat, fn):
    nat.timing(True)
    nat.timing_reset()
    try:
        fn()
        torch.cuda.synchronize()
        return nat.timing_read()
    finally:
        nat.timing(False)
        nat.timing_reset()


@pytest.mark.parametrize("Cin,Cout,K,d,T", TC_CASES)
def test_conv1d_tensor_core_path(nat, oracle, Cin, Cout, K, d, T):
    s = synth.NormalStream(6000 + Cin + Cout + K * d + T)
    B = 2
    x = s.normal((B, Cin, T))
    w = s.normal((Cout, Cin, K), 0.0, 0.02)
    b = s.normal((Cout,), 0.0, 0.02)
    pad = (K * d - d) // 2
    xd, wd, bd = dev(x), dev(w), dev(b)
    out = {}
    classes = _kernel_classes(nat, lambda: out.setdefault(
        "y", nat.bv_conv1d(xd, wd, bd, d, pad)))
    assert "conv1d_tc" in classes, classes
    y = host(out["y"])
    want = oracle.conv1d(x, w, b, d, pad)
    assert rel_l2(y, want) < LAYER_TOL


@pytest.mark.parametrize("final_act", [0, 1, 2])
def test_conv1d_tensor_core_epilogue(nat, oracle, final_act):
    s = synth.NormalStream(70 + final_act)
    C, T = 160, 300
    x = s.normal((2, C, T))
    w = s.normal((C, C, 7), 0.0, 0.05)
    b = s.normal((C,), 0.0, 0.05)
    r = s.normal((2, C, T))
    y0 = s.normal((2, C, T))
    yd = dev(y0)
    nat.bv_conv1d(dev(x), dev(w), dev(b), 3, 9, residual=dev(r), scale=1.0 / 3.0,
                  accumulate=True, final_act=final_act, y=yd)
    got = host(yd).astype(np.float64)
    conv = oracle.conv1d(x, w, b, 3, 9, store_f64=True).astype(np.float64)
    want = (conv + r) * (1.0 / 3.0) + y0
    if final_act == 1:
        want = np.clip(want, -1, 1)
    elif final_act == 2:
        want = np.tanh(want)
    assert rel_l2(got, want) < LAYER_TOL


def test_conv1d_tensor_core_inplace_residual(nat, oracle):
    s = synth.NormalStream(78)
    C, T = 128, 1000
    x = s.normal((2, C, T))
    w = s.normal((C, C, 11), 0.0, 0.02)
    cur = s.normal((2, C, T))
    cd = dev(cur)
    nat.bv_conv1d(dev(x), dev(w), None, 5, 25, residual=cd, y=cd)
    want = oracle.conv1d(x, w, None, 5, 25, store_f64=True).astype(np.float64) + cur
    assert rel_l2(host(cd), want) < LAYER_TOL


# Full-size layer shapes of the MiniMax-H3 decoder, on seeded inputs,
# checked at sampled outputs.
H3_STAGES = [(768, 2001), (384, 10006), (192, 20012), (96, 40024), (48, 80048),
             (24, 160096), (12, 320192)]


@pytest.mark.parametrize("C,T", H3_STAGES)
def test_full_size_stage_layers_sampled(nat, oracle, filt, C, T):
    s = synth.NormalStream(C * 31 + T)
    B = 2
    x = s.normal((B, C, T))
    xd = dev(x)
    rng = np.random.default_rng(C)
    n = 48 if C >= 384 else 200
    pts = np.stack([rng.integers(0, B, n), rng.integers(0, C, n), rng.integers(0, T, n)], 1)
    pts = np.concatenate([pts, [[0, 0, 0], [1, C - 1, T - 1], [0, C // 2, 1], [1, 1, T - 3]]])
    for K, d in ((3, 1), (7, 3), (11, 5)):
        w = s.normal((C, C, K), 0.0, 0.02)
        b = s.normal((C,), 0.0, 0.02)
        pad = (K * d - d) // 2
        y = host(nat.bv_conv1d(xd, dev(w), dev(b), d, pad))
        want = oracle.conv1d_points(x, w, b, d, pad, pts)
        assert rel_l2(y[pts[:, 0], pts[:, 1], pts[:, 2]], want) < LAYER_TOL, (K, d)
    la, lb = s.normal((C,), 0.0, 0.1), s.normal((C,), 0.0, 0.1)
    y = host(nat.bv_activation1d(xd, dev(la), dev(lb), filt))
    want = oracle.activation1d_points(x, la, lb, pts)
    assert rel_l2(y[pts[:, 0], pts[:, 1], pts[:, 2]], want) < LAYER_TOL


@pytest.mark.parametrize("Cin,Cout,S,T", [(1536, 768, 5, 400), (768, 384, 5, 2001),
                                          (384, 192, 2, 10006), (24, 12, 2, 160096)])
def test_full_size_conv_transpose_sampled(nat, oracle, Cin, Cout, S, T):
    s = synth.NormalStream(Cin + T)
    K = 2 * S
    pad = (K - S) // 2
    x = s.normal((2, Cin, T))
    w = s.normal((Cin, Cout, K), 0.0, 0.02)
    b = s.normal((Cout,), 0.0, 0.02)
    y = host(nat.bv_conv_transpose1d(dev(x), dev(w), dev(b), S, pad))
    Tout = (T - 1) * S + K - 2 * pad
    rng = np.random.default_rng(T)
    pts = np.stack([rng.integers(0, 2, 40), rng.integers(0, Cout, 40),
                    rng.integers(0, Tout, 40)], 1)
    pts = np.concatenate([pts, [[0, 0, 0], [1, Cout - 1, Tout - 1], [0, 1, Tout - 2]]])
    want = oracle.conv_transpose1d_points(x, w, b, S, pad, pts)
    assert rel_l2(y[pts[:, 0], pts[:, 1], pts[:, 2]], want) < LAYER_TOL


# The decoder's own kernels at full H3 stage shapes, one layer at a time
# (teacher-forced: the oracle's activation of the same float input, then its
# conv at sampled outputs).  bv_act_conv1d and bv_conv_transpose1d_ws run
# the kernels bv_decode runs for these shapes: the time-major tensor-core
# conv fed by the activation's time-major output, and the transposed convs
# with all output phases in one time-major launch.
H3_TM_UNITS = [(768, 2001, 11, 5, False), (384, 10006, 7, 3, True), (192, 20012, 3, 1, False),
               (96, 40024, 11, 1, True), (48, 80048, 7, 5, False)]


@pytest.mark.parametrize("C,T,K,d,residual", H3_TM_UNITS)
def test_full_size_act_conv_time_major_sampled(nat, oracle, filt, C, T, K, d, residual):
    s = synth.NormalStream(9000 + C + K * d)
    B = 2
    x = s.normal((B, C, T))
    la, lb = s.normal((C,), 0.0, 0.1), s.normal((C,), 0.0, 0.1)
    w = s.normal((C, C, K), 0.0, 0.02)
    b = s.normal((C,), 0.0, 0.02)
    r = s.normal((B, C, T)) if residual else None
    pad = (K * d - d) // 2
    xd, wd, bd = dev(x), dev(w), dev(b)
    rd = dev(r) if residual else None
    out = {}
    classes = _kernel_classes(nat, lambda: out.setdefault("y", nat.bv_act_conv1d(
        xd, dev(la), dev(lb), filt, wd, bd, d, pad, residual=rd)))
    # the activation writes the conv's time-major operands itself
    assert "conv1d_tm_f16" in classes and "activation_tm" in classes, classes
    assert "transpose_split" not in classes, classes
    y = host(out["y"])
    h = oracle.activation1d(x, la, lb)  # the conv's input, stored as float
    rng = np.random.default_rng(C + T)
    n = 64 if C >= 384 else 200
    pts = np.stack([rng.integers(0, B, n), rng.integers(0, C, n), rng.integers(0, T, n)], 1)
    pts = np.concatenate([pts, [[0, 0, 0], [1, C - 1, T - 1], [0, C // 2, 1], [1, 1, T - 3],
                                [0, C - 1, 127], [1, 0, 128], [0, 31, 255], [1, 32, 256]]])
    want = oracle.conv1d_points(h, w, b, d, pad, pts)
    if residual:
        want = want + r[pts[:, 0], pts[:, 1], pts[:, 2]].astype(np.float64)
    assert rel_l2(y[pts[:, 0], pts[:, 1], pts[:, 2]], want) < LAYER_TOL


@pytest.mark.parametrize("Cin,Cout,S,T", [(1536, 768, 5, 400), (768, 384, 5, 2001),
                                          (384, 192, 2, 10006), (96, 48, 2, 40024)])
def test_full_size_conv_transpose_time_major_sampled(nat, oracle, Cin, Cout, S, T):
    s = synth.NormalStream(11000 + Cin + T)
    K = 2 * S
    pad = (K - S) // 2
    x = s.normal((2, Cin, T))
    w = s.normal((Cin, Cout, K), 0.0, 0.02)
    b = s.normal((Cout,), 0.0, 0.02)
    xd, wd, bd = dev(x), dev(w), dev(b)
    out = {}
    classes = _kernel_classes(nat, lambda: out.setdefault(
        "y", nat.bv_conv_transpose1d_ws(xd, wd, bd, S, pad)))
    # every Cin here is a multiple of 8 from 48 up: the fp16 split
    assert "conv_transpose1d_tm_f16" in classes, classes
    y = host(out["y"])
    Tout = (T - 1) * S + K - 2 * pad
    assert y.shape == (2, Cout, Tout)
    rng = np.random.default_rng(T + 1)
    pts = np.stack([rng.integers(0, 2, 60), rng.integers(0, Cout, 60),
                    rng.integers(0, Tout, 60)], 1)
    pts = np.concatenate([pts, [[0, 0, 0], [1, Cout - 1, Tout - 1], [0, 1, Tout - 2],
                                [1, Cout // 2, S * 128 - 1], [0, 3, S * 256 + 1]]])
    want = oracle.conv_transpose1d_points(x, w, b, S, pad, pts)
    assert rel_l2(y[pts[:, 0], pts[:, 1], pts[:, 2]], want) < LAYER_TOL


@pytest.mark.parametrize("B,C,T", [(2, 32, 1), (1, 32, 2), (2, 32, 129), (3, 48, 130),
                                   (2, 64, 257), (1, 32, 1000), (2, 96, 4099), (1, 56, 300)])
def test_act_conv_time_major_activation_ragged(nat, oracle, filt, B, C, T):
    """The activation writing the time-major planes, both team shapes (32,
    64, 96 channels: 32-channel groups of one 16-warp team; 48 and 56: 8-channel
    groups, 56 being seven groups with the conv's second 32-channel block
    zero-padded) on ragged and tiny time axes (replicate padding at both ends
    of a tile), odd batch counts and teams that own less than one channel
    group; every output."""
    s = synth.NormalStream(13000 + B + C + T)
    x = s.normal((B, C, T), 0.0, 1.5)
    la, lb = s.normal((C,), 0.0, 0.3), s.normal((C,), 0.0, 0.3)
    Cout, K, d = 64, 7, 1
    w = s.normal((Cout, C, K), 0.0, 0.05)
    b = s.normal((Cout,), 0.0, 0.05)
    xd = dev(x)
    out = {}
    classes = _kernel_classes(nat, lambda: out.setdefault("y", nat.bv_act_conv1d(
        xd, dev(la), dev(lb), filt, dev(w), dev(b), d, 3)))
    assert "activation_tm" in classes and _has_tm(classes), classes
    assert ("conv1d_tm_f16" in classes) == (C >= 48), classes
    y = host(out["y"])
    want = oracle.conv1d(oracle.activation1d(x, la, lb), w, b, d, 3)
    assert y.shape == want.shape
    assert rel_l2(y, want) < LAYER_TOL
    np.testing.assert_allclose(y, want, rtol=1e-4, atol=1e-5)


@pytest.mark.parametrize("C,T,K,d", [(64, 777, 7, 3), (128, 300, 3, 1), (24, 513, 11, 5),
                                     (100, 257, 5, 2), (96, 1000, 1, 1), (64, 515, 1, 1),
                                     (128, 1000, 11, 5), (48, 516, 3, 1), (32, 301, 11, 3)])
def test_act_conv_small_shapes_every_element(nat, oracle, filt, C, T, K, d):
    """bv_act_conv1d on every path (time-major with the fused activation for
    32 / 64 / 96 / 128 channels, one-tap convs included, time-major through a
    separate transpose for 100, the narrow FP32 kernel for 24), every output
    against the oracle.  Rows of a multiple of 4 time steps take the staged
    bulk-store output loop (48 channels: a 16-channel group past Cout; 516:
    a last time tile of 4 steps), except where the staging does not fit beside
    the weight ring (128 channels, K 11, dilation 5)."""
    s = synth.NormalStream(12000 + C + T)
    x = s.normal((2, C, T))
    la, lb = s.normal((C,), 0.0, 0.2), s.normal((C,), 0.0, 0.2)
    w = s.normal((C, C, K), 0.0, 0.05)
    b = s.normal((C,), 0.0, 0.05)
    pad = (K * d - d) // 2
    y = host(nat.bv_act_conv1d(dev(x), dev(la), dev(lb), filt, dev(w), dev(b), d, pad))
    want = oracle.conv1d(oracle.activation1d(x, la, lb), w, b, d, pad)
    assert rel_l2(y, want) < LAYER_TOL


# -------------------------------------------------------------- AMP block


def _amp_tensors(layout, flat):
    out, off = {}, 0
    for name, shape, _ in layout:
        n = int(np.prod(shape))
        out[name] = dev(flat[off:off + n].reshape(shape))
        off += n
    return out


def test_amp_block_workload_matches_oracle(nat, oracle, filt):
    w = synth.AMP_BLOCK_C32
    x, flat = w.make()
    tens = _amp_tensors(w.layout(), flat)
    p = nat.amp_params(w.kernel, w.dilations, tens, filt)
    y = host(nat.bv_amp_block(dev(x), p))
    want = oracle.amp_block(x, flat, w.kernel, w.dilations)
    assert rel_l2(y, want) < LAYER_TOL


# (C, T, K, dilations, whether the time-major tensor-core conv qualifies)
AMP_SHAPES = [(12, 3001, 11, (1, 3, 5), False), (96, 517, 7, (1, 3, 5), True),
              (130, 64, 3, (2,), False), (16, 5, 7, (1, 3, 5, 7), False),
              (128, 2001, 11, (1, 3, 5), True), (48, 1003, 7, (1, 3, 5), True),
              (64, 300, 3, (1, 3, 5), True), (256, 130, 11, (5,), True),
              (24, 700, 11, (1, 3, 5), False), (96, 516, 7, (1, 3, 5), True),
              (32, 520, 7, (1, 3, 5), True)]


@pytest.mark.parametrize("tensor_core", [False, True])
@pytest.mark.parametrize("C,T,K,dils,tm", AMP_SHAPES)
def test_amp_block_shapes(nat, oracle, filt, C, T, K, dils, tm, tensor_core):
    """The AMP block (scale 0.5 accumulated onto y) against the oracle, with
    its convs on [B, C, T] operands or, given the larger workspace, time-major
    on the tensor cores (48 channels: a zero-padded channel block)."""
    wl = synth.AmpWorkload("t", 2, C, T, K, dils, seed=C + T)
    x, flat = wl.make()
    tens = _amp_tensors(wl.layout(), flat)
    p = nat.amp_params(K, dils, tens, filt)
    y0 = synth.NormalStream(5).normal((2, C, T))
    yd = dev(y0)
    classes = _kernel_classes(nat, lambda: nat.bv_amp_block(dev(x), p, y=yd, scale=0.5,
                                                            accumulate=True,
                                                            tensor_core=tensor_core))
    assert _has_tm(classes) == (tm and tensor_core), classes
    want = 0.5 * oracle.amp_block(x, flat, K, dils).astype(np.float64) + y0
    assert rel_l2(host(yd), want) < LAYER_TOL


# ----------------------------------------------------------------- decoder


def _decoder(nat, geo, params, filt, tile=0, overlap=0):
    return nat.Decoder(geo, params, filt=host(filt), tile_frames=tile, overlap_frames=overlap)


@pytest.mark.parametrize("final_act", ["none", "clamp", "tanh"])
def test_tiny_decoder_matches_oracle(nat, oracle, filt, final_act):
    geo = synth.tiny_geometry(final_act=final_act)
    s = synth.NormalStream(8)
    z = s.normal((2, geo.in_channels, 9))
    params = s.normal((synth.param_count(geo),), 0.0, 0.1)
    dec = _decoder(nat, geo, params, filt)
    y = host(dec.decode(dev(z)))
    want = oracle.decode(geo, params, z)
    assert y.shape == want.shape == (2, 1, 9 * geo.hop)
    assert rel_l2(y, want) < WAVE_TOL


@pytest.mark.parametrize("wname,frames", [("h3_decoder_10s_stereo", 3),
                                          ("ltx_vocoder_500f_stereo", 4)])
def test_real_geometry_short_latent(nat, oracle, filt, wname, frames):
    """The full-size channel plan of each decoder on a few latent frames,
    checked over the whole waveform (every layer kind and stride at its real
    channel count)."""
    w = synth.DECODER_WORKLOADS[wname]
    z, params = w.make()
    z = np.ascontiguousarray(z[..., :frames])
    dec = _decoder(nat, w.geometry, params, filt)
    y = host(dec.decode(dev(z)))
    want = oracle.decode(w.geometry, params, z)
    assert y.shape == want.shape
    assert rel_l2(y, want) < WAVE_TOL


@pytest.mark.parametrize("frames", [1, 2, 5, 27])
def test_decoder_tensor_core_stages(nat, oracle, filt, frames):
    """A decoder wide enough that its ConvT stages (both stride parities) and
    its AMP convs take the time-major tensor-core path (128, 96 and 48
    channels, the last with a zero-padded channel block), on short and ragged
    latents."""
    geo = synth.tiny_geometry(pre_channels=256, up_channels=(128, 96, 48), in_channels=16)
    s = synth.NormalStream(40 + frames)
    z = s.normal((2, geo.in_channels, frames))
    params = s.normal((synth.param_count(geo),), 0.0, 0.02)  # the workloads' weight scale
    dec = _decoder(nat, geo, params, filt)
    zd = dev(z)
    out = {}
    classes = _kernel_classes(nat, lambda: out.setdefault("y", dec.decode(zd)))
    assert "conv_transpose1d_tm_f16" in classes, classes
    # the 128/96/48-channel AMP convs run time-major, fed by the activation
    # writing their operand planes; the ConvT inputs are transposed
    assert _has_tm(classes) and "activation_tm" in classes, classes
    assert "transpose_split" in classes, classes
    want = oracle.decode(geo, params, z)
    assert rel_l2(host(out["y"]), want) < WAVE_TOL


def test_decoder_batch_independence_and_determinism(nat, filt):
    geo = synth.tiny_geometry()
    s = synth.NormalStream(12)
    z = s.normal((3, geo.in_channels, 7))
    params = s.normal((synth.param_count(geo),), 0.0, 0.1)
    dec = _decoder(nat, geo, params, filt)
    y = host(dec.decode(dev(z)))
    y2 = host(dec.decode(dev(z)))
    np.testing.assert_array_equal(y, y2)
    for b in range(3):
        np.testing.assert_array_equal(host(dec.decode(dev(z[b:b + 1]))), y[b:b + 1])


def test_tiled_decoder_matches_oracle(nat, oracle, filt):
    geo = synth.tiny_geometry()
    s = synth.NormalStream(13)
    z = s.normal((2, geo.in_channels, 23))
    params = s.normal((synth.param_count(geo),), 0.0, 0.1)
    for tile, ov in ((6, 2), (5, 1), (23, 4), (30, 3), (8, 0)):
        dec = _decoder(nat, geo, params, filt, tile, ov)
        y = host(dec.decode(dev(z)))
        want, _ = oracle.decode_tiled(geo, params, z, tile, ov)
        assert rel_l2(y, want) < WAVE_TOL, (tile, ov)


def test_decode_host_matches_device(nat, filt):
    geo = synth.tiny_geometry()
    s = synth.NormalStream(14)
    z = s.normal((2, geo.in_channels, 5))
    params = s.normal((synth.param_count(geo),), 0.0, 0.1)
    dec = _decoder(nat, geo, params, filt)
    yd = host(dec.decode(dev(z)))
    zh = torch.from_numpy(z).pin_memory()
    yh = torch.empty((2, 1, 5 * geo.hop), dtype=torch.float32).pin_memory()
    dec.decode_host(zh, yh)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(yh.numpy(), yd)


def test_decode_in_cuda_graph(nat, filt):
    geo = synth.tiny_geometry()
    s = synth.NormalStream(15)
    z = dev(s.normal((2, geo.in_channels, 5)))
    params = s.normal((synth.param_count(geo),), 0.0, 0.1)
    dec = _decoder(nat, geo, params, filt)
    ref = host(dec.decode(z))
    y = torch.empty((2, 1, 5 * geo.hop), device="cuda")
    ws = dec.workspace(2, 5)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dec.decode(z, y=y, workspace=ws)
    y.zero_()
    g.replay()
    np.testing.assert_array_equal(host(y), ref)


def test_decode_from_two_threads_on_two_streams(nat, filt):
    """Two host threads decode different latents at the same time, each on its
    own stream (the AMP blocks of both share the library's per-device
    streams); each result equals its single-threaded decode bit for bit."""
    import threading

    geo = synth.tiny_geometry(pre_channels=256, up_channels=(128, 96, 48), in_channels=16)
    s = synth.NormalStream(16)
    params = s.normal((synth.param_count(geo),), 0.0, 0.02)
    zs = [dev(s.normal((2, geo.in_channels, 9))), dev(s.normal((2, geo.in_channels, 9)))]
    decs = [_decoder(nat, geo, params, filt), _decoder(nat, geo, params, filt)]
    want = [host(d.decode(z)) for d, z in zip(decs, zs)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [torch.empty((2, 1, 9 * geo.hop), device="cuda") for _ in range(2)]
    wss = [decs[k].workspace(2, 9) for k in range(2)]
    torch.cuda.synchronize()
    errors = []

    def run(k):
        try:
            with torch.cuda.stream(streams[k]):
                for _ in range(20):
                    decs[k].decode(zs[k], y=outs[k], workspace=wss[k], stream=streams[k])
        except Exception as e:  # noqa: BLE001 - reported below
            errors.append(e)

    threads = [threading.Thread(target=run, args=(k,)) for k in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    torch.cuda.synchronize()
    assert not errors, errors
    for k in range(2):
        np.testing.assert_array_equal(host(outs[k]), want[k])


def test_decode_units_and_stitch_equal_the_tiled_decode(nat, filt):
    """The unit decode and stitch behind a sharded decode: each emulated rank
    decodes its contiguous range of (tile, side) units, the rows are laid
    side by side as the all-gather would, and the stitch reproduces bv_decode
    bit for bit -- tiled (two tile lengths) and untiled (units = sides)."""
    from bigvgan_waveform_decoder_alias_b200 import sharded

    geo = synth.tiny_geometry(pre_channels=256, up_channels=(128, 96, 48), in_channels=16)
    s = synth.NormalStream(17)
    B, F = 2, 23
    z = dev(s.normal((B, geo.in_channels, F)))
    params = s.normal((synth.param_count(geo),), 0.0, 0.02)
    for tile, ov in ((6, 2), (0, 0)):
        dec = _decoder(nat, geo, params, filt, tile, ov)
        want = host(dec.decode(z))
        n_units = dec.tile_count(F) * B
        assert n_units == (B * 6 if tile else B)
        P = dec.unit_length(F)
        assert P == (tile if tile else F) * geo.hop
        for world in (1, 2, 3, 5):
            ranges, per = sharded.unit_ranges(n_units, world)
            rows = torch.full((world * per, 1, P), float("nan"), device="cuda")
            for r, (a, b) in enumerate(ranges):
                if b > a:
                    dec.decode_units(z, a, b, y_units=rows[r * per:r * per + (b - a)])
            y = host(dec.stitch_units(rows[:n_units], B, F))
            np.testing.assert_array_equal(y, want)
        with pytest.raises(nat.BVError) as e:
            dec.decode_units(z, 0, n_units + 1)
        assert e.value.status == 2
        with pytest.raises(nat.BVError):
            dec.decode_units(z, 3, 3)


# ------------------------------------------------------ latent front end (H3)


@pytest.mark.parametrize("C,S,T,Cout", [(32, 2, 400, 32), (5, 3, 7, 13), (64, 2, 1, 32),
                                        (16, 1, 1000, 9)])
def test_latent_front_end_matches_oracle(nat, oracle, C, S, T, Cout):
    s = synth.NormalStream(14000 + C + S + T)
    z = s.normal((C, S, T))
    mean, std = s.normal((C,), 0.0, 0.5), np.abs(s.normal((C,), 1.0, 0.3)) + 0.1
    w = s.normal((Cout, C, 1), 0.0, 0.2)
    b = s.normal((Cout,), 0.0, 0.1)
    got = host(nat.bv_latent_front_end(dev(z), dev(mean), dev(std), dev(w), dev(b)))
    want = oracle.latent_front_end(z, mean, std, w, b)
    assert got.shape == want.shape == (S, Cout, T)
    assert rel_l2(got, want) < LAYER_TOL
    np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-6)


def test_decoder_with_latent_front_end(nat, oracle, filt):
    """bv_decode taking normalised stereo latents [C_lat, 2, frames] through
    the front end: against the oracle's front end then decode, untiled and
    tiled, and the unit decode (sharding) bit for bit against bv_decode."""
    from bigvgan_waveform_decoder_alias_b200 import sharded

    geo = synth.tiny_geometry()
    s = synth.NormalStream(18)
    Clat, B, F = 12, 2, 13
    z = s.normal((Clat, B, F))
    mean, std = s.normal((Clat,), 0.0, 0.3), np.abs(s.normal((Clat,), 1.0, 0.2)) + 0.1
    w_in = s.normal((geo.in_channels, Clat, 1), 0.0, 0.3)
    b_in = s.normal((geo.in_channels,), 0.0, 0.05)
    params = s.normal((synth.param_count(geo),), 0.0, 0.1)
    fe = (mean, std, w_in, b_in)
    zin = oracle.latent_front_end(z, mean, std, w_in, b_in)
    for tile, ov in ((0, 0), (5, 1)):
        dec = nat.Decoder(geo, params, filt=host(filt), tile_frames=tile, overlap_frames=ov,
                          front_end=fe)
        zd = dev(z)
        y = host(dec.decode(zd))
        if tile:
            want, _ = oracle.decode_tiled(geo, params, zin, tile, ov)
        else:
            want = oracle.decode(geo, params, zin)
        assert y.shape == want.shape == (B, 1, F * geo.hop)
        assert rel_l2(y, want) < WAVE_TOL, tile
        n_units = dec.tile_count(F) * B
        ranges, per = sharded.unit_ranges(n_units, 2)
        rows = torch.empty((2 * per, 1, dec.unit_length(F)), device="cuda")
        for r, (a, b_) in enumerate(ranges):
            dec.decode_units(zd, a, b_, y_units=rows[r * per:r * per + (b_ - a)])
        np.testing.assert_array_equal(host(dec.stitch_units(rows[:n_units], B, F)), y)


# ------------------------------------------------------ Music-3 DAV decoder


def _dav_params(geo, seed, std=0.2):
    s = synth.NormalStream(seed)
    params = s.normal((synth.dav_param_count(geo),), 0.0, std)
    off = 0
    for name, shape, _ in synth.dav_param_layout(geo):
        n = int(np.prod(shape))
        if name.endswith(".alpha"):  # plain Snake alphas, used as stored: near 1
            params[off:off + n] = 1.0 + 0.1 * np.tanh(params[off:off + n])
        off += n
    return params


@pytest.mark.parametrize("final_act", ["none", "tanh"])
def test_dav_tiny_matches_oracle(nat, oracle, final_act):
    geo = synth.tiny_dav_geometry(final_act=final_act)
    # weight scale 0.1: pre-tanh values of order 1, so tanh does not saturate
    # into a comparison of a few zero crossings
    params = _dav_params(geo, 50, std=0.1)
    z = synth.NormalStream(51).normal((2, geo.latent_channels, 7))
    dec = nat.DavDecoder(geo, params)
    y = host(dec.decode(dev(z)))
    want = oracle.dav_decode(geo, params, z)
    assert y.shape == want.shape == (2, 1, 7 * geo.hop)
    assert rel_l2(y, want) < WAVE_TOL


@pytest.mark.parametrize("frames", [1, 4, 9])
def test_dav_tensor_core_stages(nat, oracle, frames):
    """A DAV decoder wide enough that its Snake writes the time-major planes
    of the transposed convs and of the units' convs (the 192-channel stage's
    one-tap convs included) on the tensor cores."""
    geo = synth.tiny_dav_geometry(latent_channels=16, in_channels=16, pre_channels=384,
                                  up_channels=(192, 96, 64))
    params = _dav_params(geo, 52, std=0.05)
    z = synth.NormalStream(53 + frames).normal((2, geo.latent_channels, frames))
    dec = nat.DavDecoder(geo, params)
    zd = dev(z)
    out = {}
    classes = _kernel_classes(nat, lambda: out.setdefault("y", dec.decode(zd)))
    assert {"conv1d_tm", "conv_transpose1d_tm", "snake_split"} <= set(classes), classes
    want = oracle.dav_decode(geo, params, z)
    assert rel_l2(host(out["y"]), want) < WAVE_TOL


def test_dav_music3_geometry_short_latent(nat, oracle):
    """The full Music-3 channel plan (1536 wide, strides 8, 8, 4, 2) on a
    short stereo latent at the workloads' weight scale: 512 samples per frame
    per side, against the oracle."""
    geo = synth.MUSIC3_DAV
    s = synth.NormalStream(54)
    z = s.normal((2, geo.latent_channels, 3))
    params = synth.draw_dav_params(s, geo)
    dec = nat.DavDecoder(geo, params)
    y = host(dec.decode(dev(z)))
    want = oracle.dav_decode(geo, params, z)
    assert y.shape == (2, 1, 3 * 512)
    assert rel_l2(y, want) < WAVE_TOL
    assert np.abs(y).max() <= 1.0 and np.abs(y[0] - y[1]).max() > 0


# ------------------------------------------ LTX bandwidth-extension tail


@pytest.mark.parametrize("n_fft,hop,T", [(512, 80, 1600), (128, 80, 803), (512, 80, 80000)])
def test_mel_stft_matches_oracle(nat, oracle, n_fft, hop, T):
    s = synth.NormalStream(15000 + T)
    x = 0.3 * s.normal((2, T))
    basis = synth.stft_basis(n_fft)
    mel = synth.slaney_mel_basis(16000, n_fft, 64, 0.0, 8000.0)
    got = host(nat.bv_mel_stft(dev(x), dev(basis), dev(mel), hop))
    want = oracle.mel_stft(x, basis, mel, hop)
    assert got.shape == want.shape
    assert rel_l2(got, want) < LAYER_TOL
    np.testing.assert_allclose(got, want, rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("C,T,ratio", [(2, 1, 3), (2, 5, 3), (1, 300, 3), (2, 80000, 3),
                                       (3, 77, 2)])
def test_sinc_upsample_matches_oracle(nat, oracle, C, T, ratio):
    x = synth.NormalStream(16000 + T).normal((C, T))
    got = host(nat.bv_sinc_upsample(dev(x), ratio))
    want = oracle.hann_sinc_upsample(x, ratio)
    assert got.shape == want.shape == (C, ratio * T)
    assert rel_l2(got, want) < LAYER_TOL
    np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-6)


def _bwe_geometry_tiny():
    return (synth.LTX_BWE.replace(in_channels=2 * 16, pre_channels=48,
                                  up_channels=(32, 16, 16, 8, 8)),
            synth.BweSpec(in_rate=16000, ratio=3, n_fft=128, hop=80, n_mels=16, fmin=0.0,
                          fmax=8000.0))


@pytest.mark.parametrize("T", [80 * 8, 80 * 8 + 37, 81])
def test_bwe_tail_tiny_matches_oracle(nat, oracle, filt, T):
    geo, sp = _bwe_geometry_tiny()
    s = synth.NormalStream(17000 + T)
    low = 0.3 * s.normal((2, T))
    params = s.normal((synth.param_count(geo),), 0.0, 0.15)
    basis, mel = sp.bases()
    tail = nat.BweTail(geo, params, sp, basis, mel, filt=host(filt))
    y = host(tail(dev(low)))
    want = oracle.bwe_tail(geo, params, low, basis, mel, sp.hop, sp.ratio)
    assert y.shape == want.shape == (2, 3 * T)
    assert rel_l2(y, want) < WAVE_TOL
    assert np.abs(y).max() <= 1.0


def test_bwe_tail_full_geometry_short_signal(nat, oracle, filt):
    """The LTX extender's full channel plan (2 x 64 mel channels in, 512
    wide, rates 6, 5, 2, 2, 2) on 10 mel hops of stereo 16 kHz signal, the
    workloads' weight scale, against the oracle."""
    geo, sp = synth.LTX_BWE, synth.LTX_BWE_SPEC
    s = synth.NormalStream(18000)
    low = 0.3 * s.normal((2, 10 * sp.hop))
    params = synth._draw_params(s, synth.param_layout(geo))
    basis, mel = sp.bases()
    tail = nat.BweTail(geo, params, sp, basis, mel, filt=host(filt))
    out = {}
    classes = _kernel_classes(nat, lambda: out.setdefault("y", tail(dev(low))))
    assert {"mel_stft", "sinc_upsample", "conv1d_tm"} <= set(classes), classes
    want = oracle.bwe_tail(geo, params, low, basis, mel, sp.hop, sp.ratio)
    assert rel_l2(host(out["y"]), want) < WAVE_TOL


def test_decode_with_prepared_weights(nat, filt):
    """Weights split and packed once (bv_decoder_prepare): decodes then launch
    no weight split or ConvT repack, need a smaller workspace, and return
    the unprepared result bit for bit -- untiled, tiled and per unit."""
    geo = synth.tiny_geometry(pre_channels=256, up_channels=(128, 96, 48), in_channels=16)
    s = synth.NormalStream(20)
    params = s.normal((synth.param_count(geo),), 0.0, 0.02)
    z = dev(s.normal((2, geo.in_channels, 13)))
    for tile, ov in ((0, 0), (5, 1)):
        plain = _decoder(nat, geo, params, filt, tile, ov)
        want = host(plain.decode(z))
        prep = _decoder(nat, geo, params, filt, tile, ov).prepare()
        assert prep.workspace_size(2, 13) < plain.workspace_size(2, 13)
        np.testing.assert_array_equal(host(prep.decode(z)), want)
        # (with the per-kernel timers on, the blocks run in order, so only the
        # kernel classes are compared there)
        classes = _kernel_classes(nat, lambda: prep.decode(z))
        assert "weight_split" not in classes and "convt_repack" not in classes, classes
        assert _has_tm(classes) and _has_tmt(classes), classes
        n_units = prep.tile_count(13) * 2
        rows = prep.decode_units(z, 0, n_units)
        np.testing.assert_array_equal(host(prep.stitch_units(rows, 2, 13)), want)
