"""The tensor-core convs' three-product operand splits, emulated on the CPU.

A time-major conv multiplies operands split into two parts each, x = x_hi +
x_lo and W = W_hi + W_lo, and accumulates x_hi W_hi + x_hi W_lo + x_lo W_hi
(the lo x lo term is dropped).  Two splits are built: tf32 parts (hi keeps the
top 10 mantissa bits by truncation, lo = x - hi, itself truncated to tf32 when
the tensor core reads it), and fp16 parts (hi = fp16(x), lo = fp16(x - hi),
both rounded to nearest; the weights scaled by 2^12 into fp16's normal range
and the sums scaled back).  Here the products are formed in float64 from the
parts, so what is measured is the split's own error against the exact conv:
the floor under what the kernels can reach.  The numbers pin the reading that
the fp16 split keeps the f32 accuracy the 3xTF32 split is there to keep.
"""
import numpy as np

from bigvgan_waveform_decoder_alias_b200 import synth

W_SCALE = 4096.0  # kTmF16WScale in csrc/common.cuh


def tf32_trunc(v):
    u = np.asarray(v, np.float32).view(np.uint32) & np.uint32(0xFFFFE000)
    return u.view(np.float32).astype(np.float64)


def split_tf32(v):
    hi = tf32_trunc(v)
    lo = tf32_trunc((np.asarray(v, np.float64) - hi).astype(np.float32))
    return hi, lo


def split_f16(v):
    hi = np.asarray(v, np.float32).astype(np.float16).astype(np.float64)
    lo = (np.asarray(v, np.float64) - hi).astype(np.float16).astype(np.float64)
    return hi, lo


def im2col(x, K, d):
    """x [C, T] -> [T, C K] rows of the conv's reduction (zero padding)."""
    C, T = x.shape
    pad = (K * d - d) // 2
    xp = np.pad(x, ((0, 0), (pad, pad)))
    cols = np.stack([xp[:, j * d:j * d + T] for j in range(K)], 2)  # [C, T, K]
    return cols.transpose(1, 0, 2).reshape(T, C * K)


def split_error(X, W, split, w_scale=1.0):
    ref = X @ W.T
    xh, xl = split(X)
    wh, wl = split(W * w_scale)
    got = (xh @ wh.T + xh @ wl.T + xl @ wh.T) / w_scale
    return float(np.linalg.norm(got - ref) / np.linalg.norm(ref))


def case(C, T, K, d, x_scale, seed):
    s = synth.NormalStream(seed)
    x = (x_scale * s.normal((C, T))).astype(np.float32).astype(np.float64)
    w = s.normal((C, C, K), 0.0, 0.02).astype(np.float32).astype(np.float64)
    return im2col(x, K, d), w.reshape(C, C * K)


def test_fp16_split_error_is_below_the_tf32_split():
    for C, T, K, d in ((384, 600, 7, 3), (96, 1200, 11, 5), (48, 2000, 3, 1)):
        X, W = case(C, T, K, d, 1.0, 700 + C)
        e16 = split_error(X, W, split_f16, W_SCALE)
        e32 = split_error(X, W, split_tf32)
        assert e16 < 2e-7, (C, K, e16)
        assert e32 < 8e-7, (C, K, e32)
        assert e16 < e32, (C, K, e16, e32)


def test_fp16_split_on_small_activations():
    """Inputs of order 0.05: x_lo falls below fp16's normal range (6.1e-5)
    and keeps fewer bits, but the split stays within the tf32 split's bound."""
    X, W = case(192, 800, 7, 1, 0.05, 811)
    assert split_error(X, W, split_f16, W_SCALE) < 8e-7


def test_unscaled_fp16_weights_lose_precision():
    """Without the 2^12 scale, weights of order 0.02 leave their lo part in
    fp16's subnormals: the split error grows several-fold (the reason the
    kernels scale the weights)."""
    X, W = case(192, 800, 7, 1, 1.0, 812)
    scaled = split_error(X, W, split_f16, W_SCALE)
    unscaled = split_error(X, W, split_f16, 1.0)
    assert unscaled > 4 * scaled, (scaled, unscaled)


def test_dropped_term_matters():
    """The lo x hi product is needed: two products leave a far larger error
    (a plausible slip in a kernel's MMA sequence would show here)."""
    X, W = case(96, 600, 3, 1, 1.0, 813)
    ref = X @ W.T
    xh, xl = split_f16(X)
    wh, wl = split_f16(W * W_SCALE)
    two = (xh @ wh.T + xh @ wl.T) / W_SCALE
    err = float(np.linalg.norm(two - ref) / np.linalg.norm(ref))
    assert err > 1e-5, err
