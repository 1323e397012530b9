"""Pins of the parity oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: values the
pages print, closed forms, library routines that compute the same textbook
operation (scipy's Kaiser design, torch's convolutions in float64), invariants
and brute force on tiny inputs.  A plausible slip in the oracle -- a dropped
term, a wrong sign or index, a transposed operand, a wrong pad or trim --
fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import scipy.signal
import scipy.special
import torch
import torch.nn.functional as F

from bigvgan_waveform_decoder_alias_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


# ------------------------------------------------------------------ filter


def test_bessel_i0_page_values(oracle):
    # audiovae.rs, test bessel_i0_matches_known_values
    for x, want, tol in _golden("bessel_i0.txt"):
        x, want, tol = float(x), float(want), float(tol)
        got = oracle.bessel_i0(x)
        assert abs(got - want) < tol * max(want, 1.0), (x, got, want)


def test_bessel_i0_matches_scipy(oracle):
    for x in np.linspace(0.0, 12.0, 97):
        assert oracle.bessel_i0(x) == pytest.approx(scipy.special.i0(x), rel=1e-14)


def test_sinc_matches_numpy(oracle):
    for x in np.linspace(-7.25, 7.25, 59):
        assert oracle.sinc(x) == pytest.approx(np.sinc(x), rel=1e-14, abs=1e-16)


def test_filter_page_properties(oracle):
    # audiovae.rs, test the_resampling_filter_is_the_references
    f = oracle.kaiser_sinc(0.25, 0.3, 12)
    assert f.dtype == np.float32 and f.shape == (12,)
    assert abs(float(f.sum(dtype=np.float32)) - 1.0) < 1e-6
    for i in range(6):
        assert abs(f[i] - f[11 - i]) < 1e-6
    assert abs(f[5] - f.max()) < 1e-6


def test_filter_is_scipy_kaiser_firwin(oracle):
    """The page's design is Kaiser's window method: attenuation estimate
    A = 2.285 (N - 1) pi width + 7.95 with N = k/2 and width = 4 half_width,
    beta from Kaiser's formula, a windowed sinc with cutoff 0.25 cycles per
    sample (0.5 of Nyquist) at the half-integer centre, scaled to unit DC gain.
    scipy.signal implements each of those steps independently."""
    A = scipy.signal.kaiser_atten(6, 4 * 0.3)
    beta = scipy.signal.kaiser_beta(A)
    assert A > 50 and beta == pytest.approx(4.6638, abs=1e-4)
    want = scipy.signal.firwin(12, 0.5, window=("kaiser", beta), scale=True)
    got = oracle.kaiser_sinc_f64(0.25, 0.3, 12)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-14)
    # the page's I0 pin sits at this beta
    assert oracle.bessel_i0(beta) == pytest.approx(20.2046, rel=1e-3)


def test_filter_polyphase_halves(oracle):
    """An even-length symmetric filter pairs tap j with tap k-1-j, which has the
    other parity, so the even and the odd taps each sum to one half: each
    output phase of the 2x upsampler has unit gain."""
    f = oracle.kaiser_sinc_f64()
    assert f[0::2].sum() == pytest.approx(0.5, abs=1e-15)
    assert f[1::2].sum() == pytest.approx(0.5, abs=1e-15)


def test_filter_general_lengths(oracle):
    for k, cutoff, hw in ((8, 0.25, 0.3), (16, 0.25, 0.3), (12, 0.2, 0.25), (24, 0.25, 0.1)):
        N = k // 2
        A = scipy.signal.kaiser_atten(N, 4 * hw)
        beta = scipy.signal.kaiser_beta(A)
        want = scipy.signal.firwin(k, 2 * cutoff, window=("kaiser", beta), scale=True)
        np.testing.assert_allclose(oracle.kaiser_sinc_f64(cutoff, hw, k), want, atol=1e-13)


# -------------------------------------------------------------- activation

IDENTITY_LOG_BETA = 100.0  # 1/(e^100 + eps) ~ 4e-44: the Snake term vanishes


def _sine_gain(f, omega):
    """Closed form of up(2x) -> identity -> down(2x) on a sinusoid of angular
    frequency omega (radians per input sample).  Upsampling by zero-stuffing
    and filtering with 2 f, then filtering with f and keeping every other
    sample, is the LTI system with frequency response
    A(omega/2)^2 + A(omega/2 - pi)^2, where A(w) = sum_j f_j cos(w (j - 5.5)) is
    the zero-phase amplitude of the symmetric 12-tap filter (the pads and
    trims centre both filters, so the phase is zero)."""
    j = np.arange(len(f)) - (len(f) - 1) / 2.0

    def A(w):
        return float(np.sum(f * np.cos(w * j)))

    return A(omega / 2) ** 2 + A(omega / 2 - math.pi) ** 2


def test_activation_constant_input_closed_form(oracle):
    """x == c: each polyphase branch of the up filter has gain 1/2 (times the
    ratio 2), replicate padding keeps the edges constant, so the 2x signal is
    c everywhere, SnakeBeta maps it to c + sin^2(e^alpha c)/(e^beta + eps), and
    the unit-gain down filter keeps that -- at every t, edges included."""
    C, T = 5, 37
    cs = np.array([0.3, -1.7, 2.5, math.pi / 2, math.pi / 4], np.float64)
    la = np.array([0.05, -0.2, 0.1, 0.0, math.log(2.0)], np.float32)
    lb = np.array([-0.1, 0.15, 0.0, 0.0, 0.3], np.float32)
    x = np.repeat(cs.astype(np.float32)[None, :, None], T, axis=2)
    y = oracle.activation1d(x, la, lb, store_f64=True)
    f = oracle.kaiser_sinc()  # float taps: their even/odd sums are 1/2 to ~1e-8
    for c in range(C):
        cv = float(np.float32(cs[c]))
        a, ib = math.exp(float(la[c])), 1.0 / (math.exp(float(lb[c])) + 1e-9)
        want = cv + math.sin(a * cv) ** 2 * ib
        np.testing.assert_allclose(y[0, c], want, rtol=2e-7, atol=2e-7)
    # special values: sin^2 at pi/2 is 1, at (e^ln2)(pi/4) = pi/2 is 1
    assert y[0, 3, 0] == pytest.approx(math.pi / 2 + 1.0 / (1.0 + 1e-9), rel=1e-6)
    assert y[0, 4, 0] == pytest.approx(math.pi / 4 + 1.0 / (math.exp(float(lb[4])) + 1e-9),
                                       rel=1e-6)
    del f


def test_activation_sine_response_closed_form(oracle):
    f = oracle.kaiser_sinc().astype(np.float64)
    T = 512
    t = np.arange(T)
    C = 4
    omegas = [0.02, 0.1, 0.4, 1.1]
    phis = [0.3, -1.0, 2.0, 0.7]
    x = np.stack([np.cos(w * t + p) for w, p in zip(omegas, phis)])[None].astype(np.float32)
    la = np.zeros(C, np.float32)
    lb = np.full(C, IDENTITY_LOG_BETA, np.float32)
    y = oracle.activation1d(x, la, lb, store_f64=True)
    for c, w in enumerate(omegas):
        H = _sine_gain(oracle.kaiser_sinc().astype(np.float64), w)
        inner = slice(24, T - 24)
        np.testing.assert_allclose(y[0, c, inner], H * x[0, c, inner].astype(np.float64),
                                   atol=2e-6)
    # A band-limited sine passes unchanged to 1e-4 at low frequency ...
    w_pass = 0.02
    assert abs(_sine_gain(f, w_pass) - 1.0) < 1e-4
    inner = slice(24, T - 24)
    err = np.abs(y[0, 0, inner] - x[0, 0, inner]).max()
    assert err < 1e-4
    # ... while the cascade is a lowpass: at the input's Nyquist frequency the
    # two images each pass at half power (a half-band design), so the gain is
    # close to one half, not one
    assert abs(_sine_gain(f, math.pi) - 0.5) < 0.01
    assert abs(_sine_gain(f, 0.05) - 1.0) < 1e-4 < abs(_sine_gain(f, 0.1) - 1.0)


def test_activation_ramp_passes_interior(oracle):
    """A zero-phase unit-DC-gain LTI system maps a ramp to itself."""
    T = 200
    x = (0.01 * np.arange(T, dtype=np.float64) - 0.7).astype(np.float32)[None, None]
    y = oracle.activation1d(x, np.zeros(1, np.float32),
                            np.full(1, IDENTITY_LOG_BETA, np.float32), store_f64=True)
    np.testing.assert_allclose(y[0, 0, 12:-12], x[0, 0, 12:-12], atol=1e-6)
    # at the edges replicate padding bends the ramp towards the edge value
    assert abs(y[0, 0, 0] - x[0, 0, 0]) > 1e-4


def _torch_activation(x, la, lb, f, eps=1e-9):
    """The pages' activation written with torch's own float64 operators."""
    x = torch.as_tensor(x, dtype=torch.float64)
    C = x.shape[1]
    f = torch.as_tensor(f, dtype=torch.float64)
    K = f.numel()
    pad = K // 2 - 1
    wk = f.view(1, 1, K).expand(C, 1, K).contiguous()
    xp = F.pad(x, (pad, pad), mode="replicate")
    u = 2.0 * F.conv_transpose1d(xp, wk, stride=2, groups=C)
    pl = pad * 2 + (K - 2) // 2
    pr = pad * 2 + (K - 2 + 1) // 2
    u = u[..., pl:u.shape[-1] - pr]
    a = torch.exp(torch.as_tensor(la, dtype=torch.float64)).view(1, C, 1)
    ib = 1.0 / (torch.exp(torch.as_tensor(lb, dtype=torch.float64)).view(1, C, 1) + eps)
    v = u + torch.sin(a * u) ** 2 * ib
    vp = F.pad(v, (K // 2 - 1, K // 2), mode="replicate")
    return F.conv1d(vp, wk, stride=2, groups=C).numpy()


@pytest.mark.parametrize("T", [1, 2, 3, 7, 13, 64])
def test_activation_matches_torch_composition(oracle, T):
    s = synth.NormalStream(11 + T)
    B, C = 2, 3
    x = s.normal((B, C, T), 0.0, 2.0)
    la, lb = s.normal((C,), 0.0, 0.3), s.normal((C,), 0.0, 0.3)
    f = oracle.kaiser_sinc()
    y = oracle.activation1d(x, la, lb, store_f64=True)
    want = _torch_activation(x, la, lb, f)
    assert y.shape == (B, C, T)
    np.testing.assert_allclose(y, want, rtol=1e-6, atol=1e-6)


def test_activation_points_match_rows(oracle):
    s = synth.NormalStream(5)
    x = s.normal((2, 3, 300))
    la, lb = s.normal((3,), 0.0, 0.1), s.normal((3,), 0.0, 0.1)
    y = oracle.activation1d(x, la, lb, store_f64=True)
    pts = [(0, 0, 0), (1, 2, 299), (0, 1, 150), (1, 0, 3), (0, 2, 296), (1, 1, 97)]
    got = oracle.activation1d_points(x, la, lb, pts)
    want = [y[b, c, t] for b, c, t in pts]
    np.testing.assert_allclose(got, want, rtol=1e-7, atol=1e-7)


def test_activation_f32_store_is_rounding_close(oracle):
    s = synth.NormalStream(9)
    x = s.normal((1, 4, 500))
    la, lb = s.normal((4,), 0.0, 0.1), s.normal((4,), 0.0, 0.1)
    y32 = oracle.activation1d(x, la, lb, store_f64=False).astype(np.float64)
    y64 = oracle.activation1d(x, la, lb, store_f64=True).astype(np.float64)
    rel = np.linalg.norm(y32 - y64) / np.linalg.norm(y64)
    assert 0 < rel < 1e-6


# ------------------------------------------------------------------ convs

CONV_CASES = [(K, d, T) for K in (3, 7, 11) for d in (1, 3, 5) for T in (1, 2, 3, 7, 40)]


@pytest.mark.parametrize("K,d,T", CONV_CASES)
def test_conv1d_matches_torch_f64(oracle, K, d, T):
    s = synth.NormalStream(100 + 7 * K + 3 * d + T)
    B, Cin, Cout = 2, 3, 4
    x = s.normal((B, Cin, T))
    w = s.normal((Cout, Cin, K), 0.0, 0.5)
    b = s.normal((Cout,), 0.0, 0.5)
    pad = (K * d - d) // 2
    y = oracle.conv1d(x, w, b, dilation=d, pad=pad, store_f64=True)
    want = F.conv1d(torch.as_tensor(x, dtype=torch.float64), torch.as_tensor(w, dtype=torch.float64),
                    torch.as_tensor(b, dtype=torch.float64), padding=pad, dilation=d).numpy()
    np.testing.assert_allclose(y, want, rtol=1e-6, atol=1e-6)


def test_conv1d_is_im2col_gemm(oracle):
    """The identity the page states for its device arm: with row (i, j) of the
    column matrix holding x[i, t + j d - pad] (zero outside), the conv is
    W[out, in*k] @ col plus the bias."""
    s = synth.NormalStream(3)
    Cin, Cout, K, d, T = 5, 6, 7, 3, 50
    pad = (K * d - d) // 2
    x = s.normal((1, Cin, T))
    w = s.normal((Cout, Cin, K))
    b = s.normal((Cout,))
    col = np.zeros((Cin * K, T))
    for i in range(Cin):
        for j in range(K):
            for t in range(T):
                p = t + j * d - pad
                if 0 <= p < T:
                    col[i * K + j, t] = x[0, i, p]
    want = w.reshape(Cout, Cin * K).astype(np.float64) @ col + b[:, None]
    y = oracle.conv1d(x, w, b, dilation=d, pad=pad, store_f64=True)
    np.testing.assert_allclose(y[0], want, rtol=1e-6, atol=1e-5)


def test_conv1d_unpadded_and_no_bias(oracle):
    s = synth.NormalStream(4)
    x = s.normal((2, 3, 20))
    w = s.normal((2, 3, 5))
    y = oracle.conv1d(x, w, None, dilation=2, pad=0, store_f64=True)
    want = F.conv1d(torch.as_tensor(x, dtype=torch.float64),
                    torch.as_tensor(w, dtype=torch.float64), dilation=2).numpy()
    assert y.shape == (2, 2, 12)
    np.testing.assert_allclose(y, want, rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("s_,T", [(s_, T) for s_ in (2, 5, 6, 3) for T in (1, 2, 3, 7, 20)])
def test_conv_transpose1d_matches_torch_and_zero_stuffing(oracle, s_, T):
    rs = synth.NormalStream(200 + 10 * s_ + T)
    B, Cin, Cout = 2, 3, 4
    K = 2 * s_
    pad = (K - s_) // 2
    x = rs.normal((B, Cin, T))
    w = rs.normal((Cin, Cout, K), 0.0, 0.5)
    b = rs.normal((Cout,), 0.0, 0.5)
    y = oracle.conv_transpose1d(x, w, b, stride=s_, pad=pad, store_f64=True)
    xt = torch.as_tensor(x, dtype=torch.float64)
    wt = torch.as_tensor(w, dtype=torch.float64)
    bt = torch.as_tensor(b, dtype=torch.float64)
    want = F.conv_transpose1d(xt, wt, bt, stride=s_, padding=pad).numpy()
    assert y.shape == want.shape == (B, Cout, (T - 1) * s_ + K - 2 * pad)
    np.testing.assert_allclose(y, want, rtol=1e-6, atol=1e-6)
    # textbook identity: zero-stuff by s, pad K-1-pad each side, correlate
    # with the kernel flipped in time and transposed in channels
    Ls = (T - 1) * s_ + 1
    st = torch.zeros(B, Cin, Ls, dtype=torch.float64)
    st[..., ::s_] = xt
    wf = wt.flip(-1).transpose(0, 1).contiguous()
    alt = F.conv1d(F.pad(st, (K - 1 - pad, K - 1 - pad)), wf, bt).numpy()
    np.testing.assert_allclose(y, alt, rtol=1e-6, atol=1e-6)


def test_conv_points_match_full(oracle):
    s = synth.NormalStream(8)
    x = s.normal((2, 4, 33))
    w = s.normal((5, 4, 7))
    b = s.normal((5,))
    y = oracle.conv1d(x, w, b, dilation=3, pad=9, store_f64=True)
    pts = [(0, 0, 0), (1, 4, 32), (0, 2, 16), (1, 1, 5)]
    np.testing.assert_allclose(oracle.conv1d_points(x, w, b, 3, 9, pts),
                               [y[p] for p in pts], rtol=1e-7, atol=1e-7)
    wt = s.normal((4, 3, 10))
    bt = s.normal((3,))
    yt = oracle.conv_transpose1d(x, wt, bt, stride=5, pad=2, store_f64=True)
    pts = [(0, 0, 0), (1, 2, yt.shape[2] - 1), (0, 1, 77), (1, 0, 3)]
    np.testing.assert_allclose(oracle.conv_transpose1d_points(x, wt, bt, 5, 2, pts),
                               [yt[p] for p in pts], rtol=1e-7, atol=1e-7)


# ----------------------------------------------------------------- decoder


def _torch_decode(geo, params, z, f):
    """The decoder composed from torch float64 operators and the torch
    activation above, walking the flat parameters in module order."""
    layout = synth.param_layout(geo)
    tensors, off = {}, 0
    for name, shape, _ in layout:
        n = int(np.prod(shape))
        tensors[name] = torch.as_tensor(params[off:off + n].reshape(shape), dtype=torch.float64)
        off += n
    T = lambda a: torch.as_tensor(a, dtype=torch.float64)  # noqa: E731
    x = F.conv1d(T(z), tensors["conv_pre.w"], tensors["conv_pre.b"],
                 padding=(geo.pre_kernel - 1) // 2)
    for i, (s_, k) in enumerate(zip(geo.up_rates, geo.up_kernels)):
        x = F.conv_transpose1d(x, tensors[f"ups.{i}.w"], tensors[f"ups.{i}.b"], stride=s_,
                               padding=(k - s_) // 2)
        outs = []
        for j, kb in enumerate(geo.block_kernels):
            cur = x.clone()
            for u, d in enumerate(geo.dilations):
                p = f"stage{i}.block{j}.unit{u}"
                h = T(_torch_activation(cur.numpy(), tensors[f"{p}.act1.log_alpha"].numpy(),
                                        tensors[f"{p}.act1.log_beta"].numpy(), f))
                h = F.conv1d(h, tensors[f"{p}.conv1.w"], tensors[f"{p}.conv1.b"],
                             padding=(kb * d - d) // 2, dilation=d)
                h = T(_torch_activation(h.numpy(), tensors[f"{p}.act2.log_alpha"].numpy(),
                                        tensors[f"{p}.act2.log_beta"].numpy(), f))
                h = F.conv1d(h, tensors[f"{p}.conv2.w"], tensors[f"{p}.conv2.b"],
                             padding=(kb - 1) // 2)
                cur = cur + h
            outs.append(cur)
        x = sum(outs) / len(outs)
    x = T(_torch_activation(x.numpy(), tensors["act_post.log_alpha"].numpy(),
                            tensors["act_post.log_beta"].numpy(), f))
    y = F.conv1d(x, tensors["conv_post.w"], tensors["conv_post.b"],
                 padding=(geo.post_kernel - 1) // 2)
    if geo.final_act == "tanh":
        y = torch.tanh(y)
    elif geo.final_act == "clamp":
        y = y.clamp(-1.0, 1.0)
    return y.numpy()


def _tiny_inputs(geo, B=2, F_=6, seed=21):
    s = synth.NormalStream(seed)
    z = s.normal((B, geo.in_channels, F_))
    params = s.normal((synth.param_count(geo),), 0.0, 0.2)
    return z, params


def test_param_counts_agree(oracle):
    for geo in (synth.H3, synth.LTX, synth.tiny_geometry()):
        assert oracle.param_count(geo) == synth.param_count(geo)
        assert oracle.hop(geo) == geo.hop


@pytest.mark.parametrize("final_act", ["none", "clamp", "tanh"])
def test_decode_matches_torch_composition(oracle, final_act):
    geo = synth.tiny_geometry(final_act=final_act)
    z, params = _tiny_inputs(geo)
    f = oracle.kaiser_sinc()
    y = oracle.decode(geo, params, z, store_f64=True)
    want = _torch_decode(geo, params, z, f.astype(np.float64))
    assert want.shape[2] == oracle.raw_len(geo, z.shape[2])
    L = z.shape[2] * geo.hop
    assert y.shape == (2, 1, L)
    np.testing.assert_allclose(y, want[..., :L], rtol=1e-6, atol=1e-6)


def test_decode_geometry_and_range(oracle):
    """Output length frames x hop; the odd-stride ConvT leaves extra raw samples
    that the trim drops; finite, inside the tanh range, not silent, and the
    two sides differ."""
    geo = synth.tiny_geometry()
    assert oracle.raw_len(geo, 6) == ((6 - 1) * 5 + 10 - 4 - 1) * 4 + 4  # 5F+1, then x4
    s = synth.NormalStream(1)
    t = np.arange(6)
    z = np.stack([0.4 * np.sin(0.13 * np.arange(geo.in_channels)[:, None] + 0.7 * t + ph)
                  for ph in (0.0, 1.0)]).astype(np.float32)
    params = s.normal((synth.param_count(geo),), 0.0, 0.2)
    y = oracle.decode(geo, params, z)
    assert y.shape == (2, 1, 6 * geo.hop)
    assert np.isfinite(y).all() and np.abs(y).max() <= 1.0
    assert np.sqrt(np.mean(y.astype(np.float64) ** 2)) > 1e-4
    assert np.abs(y[0] - y[1]).max() > 0


def test_decode_residual_identity(oracle):
    """With every conv2 weight and bias zero, each residual unit adds zero, so
    each AMP block is the identity and the stage mean is the ConvT output."""
    geo = synth.tiny_geometry(final_act="none")
    z, params = _tiny_inputs(geo)
    p = params.copy()
    off = 0
    for name, shape, _ in synth.param_layout(geo):
        n = int(np.prod(shape))
        if ".conv2." in name:
            p[off:off + n] = 0.0
        off += n
    y = oracle.decode(geo, p, z, store_f64=True)
    tensors, off = {}, 0
    for name, shape, _ in synth.param_layout(geo):
        n = int(np.prod(shape))
        tensors[name] = p[off:off + n].reshape(shape)
        off += n
    x = oracle.conv1d(z, tensors["conv_pre.w"], tensors["conv_pre.b"], 1, 3, store_f64=True)
    for i, (s_, k) in enumerate(zip(geo.up_rates, geo.up_kernels)):
        x = oracle.conv_transpose1d(x, tensors[f"ups.{i}.w"], tensors[f"ups.{i}.b"], s_,
                                    (k - s_) // 2, store_f64=True)
    x = oracle.activation1d(x, tensors["act_post.log_alpha"], tensors["act_post.log_beta"],
                            store_f64=True)
    want = oracle.conv1d(x, tensors["conv_post.w"], tensors["conv_post.b"], 1, 3,
                         store_f64=True)
    # the chained layer calls hand back float tensors, so allow float rounding
    np.testing.assert_allclose(y, want[..., :y.shape[2]], rtol=1e-5, atol=2e-6)


def test_decode_batch_independence(oracle):
    geo = synth.tiny_geometry()
    z, params = _tiny_inputs(geo)
    y = oracle.decode(geo, params, z)
    for b in range(2):
        np.testing.assert_array_equal(oracle.decode(geo, params, z[b:b + 1]), y[b:b + 1])


def test_tiling_rule(oracle):
    assert oracle.tile_count(2400, 200, 16) == 13
    assert oracle.tile_count(200, 200, 16) == 1
    assert oracle.tile_count(201, 200, 16) == 2
    assert oracle.tile_count(384, 200, 16) == 2
    assert oracle.tile_count(385, 200, 16) == 3


def test_tiled_decode_identities(oracle):
    geo = synth.tiny_geometry()
    z, params = _tiny_inputs(geo, F_=13)
    y = oracle.decode(geo, params, z)
    # one tile that covers everything is the untiled decode
    yt, cnt = oracle.decode_tiled(geo, params, z, tile=13, overlap=2)
    np.testing.assert_array_equal(yt, y)
    assert (cnt == 1).all()
    # tiles of 5 frames with 2 overlapping: starts 0, 3, 6, 9 (the last 4 long)
    yt, cnt = oracle.decode_tiled(geo, params, z, tile=5, overlap=2)
    hop = geo.hop
    assert oracle.tile_count(13, 5, 2) == 4
    want_cnt = np.zeros(13 * hop)
    for st, ln in ((0, 5), (3, 5), (6, 5), (9, 4)):
        want_cnt[st * hop:(st + ln) * hop] += 1
    np.testing.assert_array_equal(cnt, want_cnt)
    # where one tile alone covers a sample, it is that tile's own decode
    y0 = oracle.decode(geo, params, z[..., 0:5])
    np.testing.assert_array_equal(yt[..., :3 * hop], y0[..., :3 * hop])
    # in an overlap, the mean of the two tiles
    y1 = oracle.decode(geo, params, z[..., 3:8])
    ov = slice(3 * hop, 5 * hop)
    want = ((y0[..., ov].astype(np.float64) + y1[..., 0:2 * hop]) / 2).astype(np.float32)
    np.testing.assert_allclose(yt[..., ov], want, rtol=0, atol=1e-7)
    # picking tiles leaves the rest uncovered
    yp, cp = oracle.decode_tiled(geo, params, z, tile=5, overlap=2, tiles=(0, 1))
    assert np.isnan(yp[..., 5 * hop:]).all() and (cp[5 * hop:] == 0).all()


# --------------------------------------------------------------- generator


def test_splitmix64_reference_words():
    for seed, idx, val in _golden("splitmix64.txt"):
        w = synth.splitmix64_words(int(seed), int(idx), 1)
        assert int(w[0]) == int(val)


def test_normal_stream_is_a_stream():
    a = synth.NormalStream(7)
    x1 = a.normal((1000,))
    x2 = a.normal((333,))
    b = synth.NormalStream(7)
    both = b.normal((1333,))
    np.testing.assert_array_equal(np.concatenate([x1, x2]), both)
    big = synth.NormalStream(3).normal((200000,)).astype(np.float64)
    assert abs(big.mean()) < 0.01 and abs(big.std() - 1.0) < 0.01


# ------------------------------------------------- latent front end (H3 decode)


def test_latent_front_end_identity_reads_the_stereo_layout(oracle):
    """std 1, mean 0 and an identity projection return the latents as they
    are, side by side: out[s, c, t] = z[c, s, t] -- the [C, 2, T] layout of
    the audiovae.rs page's `AudioVae::decode` (z[(ci 2 + ch) t + ti])."""
    rng = np.random.default_rng(5)
    C, S, T = 6, 2, 11
    z = rng.standard_normal((C, S, T)).astype(np.float32)
    w = np.eye(C, dtype=np.float32)[:, :, None]
    out = oracle.latent_front_end(z, np.zeros(C, np.float32), np.ones(C, np.float32), w, None)
    np.testing.assert_array_equal(out, z.transpose(1, 0, 2))


def test_latent_front_end_affine_denormalisation(oracle):
    """With an identity projection and a bias: out = z std + mean + bias,
    channel by channel (the de-normalisation runs before the projection)."""
    rng = np.random.default_rng(6)
    C, S, T = 5, 2, 9
    z = rng.standard_normal((C, S, T)).astype(np.float32)
    mean = rng.standard_normal(C).astype(np.float32)
    std = rng.uniform(0.5, 2.0, C).astype(np.float32)
    bias = rng.standard_normal(C).astype(np.float32)
    w = np.eye(C, dtype=np.float32)[:, :, None]
    out = oracle.latent_front_end(z, mean, std, w, bias, store_f64=True).astype(np.float64)
    lat = z.astype(np.float64) * std[:, None, None] + mean[:, None, None]
    want = lat.transpose(1, 0, 2) + bias[None, :, None]
    np.testing.assert_allclose(out, want, rtol=1e-6, atol=1e-6)


def test_latent_front_end_projection_matches_torch(oracle):
    """The projection against torch's float64 conv1d (kernel size 1) of the
    float-stored de-normalised latents."""
    import torch
    rng = np.random.default_rng(7)
    C, S, T, Cout = 8, 2, 40, 12
    z = rng.standard_normal((C, S, T)).astype(np.float32)
    mean = rng.standard_normal(C).astype(np.float32)
    std = rng.uniform(0.5, 2.0, C).astype(np.float32)
    w = (0.3 * rng.standard_normal((Cout, C, 1))).astype(np.float32)
    b = rng.standard_normal(Cout).astype(np.float32)
    out = oracle.latent_front_end(z, mean, std, w, b)
    lat = (z.astype(np.float64) * std[:, None, None] + mean[:, None, None]).astype(np.float32)
    want = torch.nn.functional.conv1d(torch.from_numpy(lat.transpose(1, 0, 2).astype(np.float64)),
                                      torch.from_numpy(w.astype(np.float64)),
                                      torch.from_numpy(b.astype(np.float64))).numpy()
    np.testing.assert_allclose(out, want.astype(np.float32), rtol=2e-6, atol=2e-6)


# ----------------------------------------------------- Music-3 DAV decoder


def test_snake_closed_forms(oracle):
    """Plain Snake x + sin^2(a x)/(a + 1e-9) at points where sin^2 is known:
    a x = pi/2 adds 1/(a + 1e-9), a x = pi adds 0, x = 0 stays 0."""
    a = np.array([0.5, 1.0, 2.0, 1.7], np.float32)
    x = np.stack([np.pi / 2 / a, np.pi / a, np.zeros(4), -np.pi / 2 / a], 1)[None].astype(
        np.float32)
    y = oracle.snake1d(x, a, store_f64=True).astype(np.float64)
    xd = x.astype(np.float64)
    ad = a.astype(np.float64)[:, None]
    want = np.stack([xd[0, :, 0] + 1 / (ad[:, 0] + 1e-9), xd[0, :, 1], np.zeros(4),
                     xd[0, :, 3] + 1 / (ad[:, 0] + 1e-9)], 1)
    np.testing.assert_allclose(y[0], want, rtol=1e-6, atol=1e-7)


def _dav_tensors(geo, params):
    out, off = {}, 0
    for name, shape, _ in synth.dav_param_layout(geo):
        n = int(np.prod(shape))
        out[name] = params[off:off + n].reshape(shape)
        off += n
    return out


def _dav_inputs(geo, B=2, F_=5, seed=41):
    s = synth.NormalStream(seed)
    z = s.normal((B, geo.latent_channels, F_))
    params = s.normal((synth.dav_param_count(geo),), 0.0, 0.2)
    t = _dav_tensors(geo, params)
    for name in t:  # plain Snake alphas are used as stored: keep them near 1
        if name.endswith(".alpha"):
            t[name][:] = 1.0 + 0.1 * np.tanh(t[name])
    return z, params


def _torch_dav(geo, params, z):
    """The DAV decoder composed from torch float64 operators."""
    t = {k: torch.as_tensor(v, dtype=torch.float64) for k, v in _dav_tensors(geo, params).items()}

    def snake(x, a):
        a = a[None, :, None]
        return x + torch.sin(a * x) ** 2 / (a + 1e-9)

    x = F.conv1d(torch.as_tensor(z, dtype=torch.float64), t["dec_in.w"], t["dec_in.b"])
    x = F.conv1d(x, t["conv_pre.w"], t["conv_pre.b"], padding=(geo.pre_kernel - 1) // 2)
    for i, (s_, k) in enumerate(zip(geo.up_rates, geo.up_kernels)):
        x = F.conv_transpose1d(snake(x, t[f"stage{i}.act.alpha"]), t[f"stage{i}.up.w"],
                               t[f"stage{i}.up.b"], stride=s_, padding=(k - s_) // 2)
        for u, d in enumerate(geo.dilations):
            p = f"stage{i}.unit{u}"
            h = snake(x, t[f"{p}.a1.alpha"])
            h = F.conv1d(h, t[f"{p}.c1.w"], t[f"{p}.c1.b"], dilation=d,
                         padding=d * (geo.unit_kernel - 1) // 2)
            h = F.conv1d(snake(h, t[f"{p}.a2.alpha"]), t[f"{p}.c2.w"], t[f"{p}.c2.b"])
            x = x + h
    x = snake(x, t["act_post.alpha"])
    y = F.conv1d(x, t["conv_post.w"], t["conv_post.b"], padding=(geo.post_kernel - 1) // 2)
    return torch.tanh(y).numpy() if geo.final_act == "tanh" else y.numpy()


def test_dav_param_counts_and_hop(oracle):
    for geo in (synth.MUSIC3_DAV, synth.tiny_dav_geometry()):
        assert oracle.dav_param_count(geo) == synth.dav_param_count(geo)
        assert oracle.dav_hop(geo) == geo.hop
    # the page's Music3Dav: 512 samples per latent frame, 44.1 kHz
    assert synth.MUSIC3_DAV.hop == 512 and synth.MUSIC3_DAV.sample_rate == 44100


@pytest.mark.parametrize("final_act", ["none", "tanh"])
def test_dav_matches_torch_composition(oracle, final_act):
    geo = synth.tiny_dav_geometry(final_act=final_act)
    z, params = _dav_inputs(geo)
    y = oracle.dav_decode(geo, params, z, store_f64=True)
    want = _torch_dav(geo, params, z)
    assert y.shape == want.shape == (2, 1, z.shape[2] * geo.hop)
    np.testing.assert_allclose(y, want, rtol=1e-6, atol=1e-6)


def test_dav_geometry_and_range(oracle):
    """The page's Music-3 vocoder test, on the small geometry: a structured
    latent (0.4 sin(0.13 c + 0.7 t) over the 2 x C stereo channels) decodes
    to frames x hop samples per side, finite, inside the tanh range, not
    silent, and the two halves differ."""
    geo = synth.tiny_dav_geometry()
    frames, C = 12, geo.latent_channels
    c = np.arange(2 * C)[:, None]
    t = np.arange(frames)[None, :]
    z = (0.4 * np.sin(c * 0.13 + t * 0.7)).reshape(2, C, frames).astype(np.float32)
    _, params = _dav_inputs(geo)
    y = oracle.dav_decode(geo, params, z)
    assert y.shape == (2, 1, frames * geo.hop)
    assert np.isfinite(y).all() and np.abs(y).max() <= 1.0
    assert np.sqrt(np.mean(y.astype(np.float64) ** 2)) > 1e-4
    assert np.abs(y[0] - y[1]).max() > 0


def test_dav_residual_identity(oracle):
    """With every unit's second conv zero, the units add nothing: the decoder
    is dec_in, conv_pre, (Snake, ConvT) per stage, Snake, conv_post."""
    geo = synth.tiny_dav_geometry(final_act="none")
    z, params = _dav_inputs(geo)
    p = params.copy()
    off = 0
    for name, shape, _ in synth.dav_param_layout(geo):
        n = int(np.prod(shape))
        if ".c2." in name:
            p[off:off + n] = 0.0
        off += n
    y = oracle.dav_decode(geo, p, z, store_f64=True)
    t = _dav_tensors(geo, p)
    x = oracle.conv1d(z, t["dec_in.w"], t["dec_in.b"], 1, 0, store_f64=True)
    x = oracle.conv1d(x, t["conv_pre.w"], t["conv_pre.b"], 1, 3, store_f64=True)
    for i, (s_, k) in enumerate(zip(geo.up_rates, geo.up_kernels)):
        x = oracle.snake1d(x, t[f"stage{i}.act.alpha"], store_f64=True)
        x = oracle.conv_transpose1d(x, t[f"stage{i}.up.w"], t[f"stage{i}.up.b"], s_,
                                    (k - s_) // 2, store_f64=True)
    x = oracle.snake1d(x, t["act_post.alpha"], store_f64=True)
    want = oracle.conv1d(x, t["conv_post.w"], t["conv_post.b"], 1, 3, store_f64=True)
    np.testing.assert_allclose(y, want, rtol=1e-5, atol=2e-6)


def test_dav_batch_independence(oracle):
    geo = synth.tiny_dav_geometry()
    z, params = _dav_inputs(geo)
    y = oracle.dav_decode(geo, params, z)
    for b in range(2):
        np.testing.assert_array_equal(oracle.dav_decode(geo, params, z[b:b + 1]), y[b:b + 1])


# ---------------------------------------------- LTX bandwidth-extension tail


def test_mel_basis_is_torchaudio_slaney():
    """The synthesised mel filterbank (an input: the checkpoint's is not
    available) equals torchaudio's Slaney-scale, Slaney-normalised bank."""
    import torchaudio
    sp = synth.LTX_BWE_SPEC
    _, mel = sp.bases()
    want = torchaudio.functional.melscale_fbanks(sp.n_fft // 2 + 1, sp.fmin, sp.fmax, sp.n_mels,
                                                 sp.in_rate, norm="slaney",
                                                 mel_scale="slaney").numpy().T
    np.testing.assert_allclose(mel, want, rtol=1e-5, atol=1e-7)


@pytest.mark.parametrize("n_fft,hop,T", [(512, 80, 1600), (128, 80, 803), (64, 16, 100)])
def test_mel_stft_matches_torch_stft(oracle, n_fft, hop, T):
    """The causal log-mel against torch.stft (periodic Hann window, no
    centring) of the signal left-padded with n_fft - hop zeros, then the mel
    bank and log(max(., 1e-5)), folded to [C n_mels, frames]."""
    rng = np.random.default_rng(n_fft + T)
    x = (0.3 * rng.standard_normal((2, T))).astype(np.float32)
    basis = synth.stft_basis(n_fft)
    mel = synth.slaney_mel_basis(16000, n_fft, 24, 0.0, 8000.0)
    got = oracle.mel_stft(x, basis, mel, hop)
    xp = torch.nn.functional.pad(torch.as_tensor(x, dtype=torch.float64), (n_fft - hop, 0))
    S = torch.stft(xp, n_fft=n_fft, hop_length=hop, win_length=n_fft,
                   window=torch.hann_window(n_fft, periodic=True, dtype=torch.float64),
                   center=False, return_complex=True).abs()
    m = torch.log(torch.clamp(torch.as_tensor(mel, dtype=torch.float64) @ S, min=1e-5))
    want = m.reshape(2 * mel.shape[0], -1).numpy()
    assert got.shape == want.shape and got.shape[1] == oracle.mel_frames(T, n_fft, hop)
    np.testing.assert_allclose(got, want, rtol=1e-5, atol=2e-5)


@pytest.mark.parametrize("T", [1, 5, 300])
def test_hann_sinc_upsample_matches_torchaudio(oracle, T):
    """x3 upsampling against torchaudio's Hann-windowed sinc resampler
    (lowpass width 6, rolloff 0.99) run on the signal extended by 10
    replicated samples each side: the page pads by replicating, torchaudio by
    zeros, so the extension makes the two agree everywhere, edges included."""
    import torchaudio
    rng = np.random.default_rng(T)
    x = rng.standard_normal((2, T)).astype(np.float32)
    got = oracle.hann_sinc_upsample(x, 3, store_f64=True).astype(np.float64)
    e = 10
    xe = np.pad(x.astype(np.float64), ((0, 0), (e, e)), mode="edge")
    ref = torchaudio.functional.resample(torch.as_tensor(xe), 1, 3, lowpass_filter_width=6,
                                         rolloff=0.99,
                                         resampling_method="sinc_interp_hann").numpy()
    want = ref[:, 3 * e:3 * e + 3 * T]
    assert got.shape == (2, 3 * T)
    # the page rounds its taps to float: about 6e-8 of the sum of |taps| x |x|
    np.testing.assert_allclose(got, want, rtol=1e-6, atol=1e-6)


def _bwe_tiny():
    geo = synth.LTX_BWE.replace(in_channels=2 * 16, pre_channels=48,
                                up_channels=(32, 16, 16, 8, 8))
    return geo, synth.BweSpec(in_rate=16000, ratio=3, n_fft=128, hop=80, n_mels=16, fmin=0.0,
                              fmax=8000.0)


def test_bwe_tail_is_its_composition(oracle):
    """clamp(extender(log-mel(padded low)) + upsample(padded low)) over the
    first 3 T samples, against the oracle's own steps: the low signal zero
    padded to whole mel hops, the mel front end, one decode of the folded
    stereo mel (2 outputs, no final op), the x3 skip, the clamped sum."""
    geo, sp = _bwe_tiny()
    s = synth.NormalStream(61)
    T = 8 * sp.hop + 37  # not a whole number of hops
    low = 0.3 * s.normal((2, T))
    params = s.normal((synth.param_count(geo),), 0.0, 0.15)
    basis, mel = sp.bases()
    y = oracle.bwe_tail(geo, params, low, basis, mel, sp.hop, sp.ratio)
    Tp = -(-T // sp.hop) * sp.hop
    padded = np.zeros((2, Tp), np.float32)
    padded[:, :T] = low
    m = oracle.mel_stft(padded, basis, mel, sp.hop)
    res = oracle.decode(geo, params, m[None])[0]
    skip = oracle.hann_sinc_upsample(padded, sp.ratio)
    want = np.clip(res[:, :3 * T].astype(np.float64) + skip[:, :3 * T], -1.0, 1.0)
    assert y.shape == (2, 3 * T)
    np.testing.assert_allclose(y, want, rtol=1e-6, atol=1e-7)
    assert np.abs(y).max() <= 1.0 and np.abs(res).max() > 0
