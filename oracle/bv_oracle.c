/*
 * bv_oracle.c -- the parity oracle for the BigVGAN alias-free decoder.
 *
 * TEST INFRASTRUCTURE, NOT THE PRODUCT.  Only the test suite, the smoke check
 * and the bench's CPU-baseline leg may load or call this file.  It shares no
 * code, header, table or constant with the CUDA library and imports nothing
 * from it.
 *
 * What it is: a plain, slow, single-threaded C statement of the decoder as the
 * pages define it, with every dot product and FIR accumulated in double and
 * libm's double exp/sin/tanh.  Each tensor that the pages store between
 * operations (a layer output) is rounded to float when `store_f64` is 0, which
 * matches the pages' "f32 throughout" rule; with `store_f64` = 1 everything
 * stays double (used to study error growth).
 *
 * Sources (all Rust, on the pages):
 *   [H3]  docs.rs cortiq-engine 0.5.74, src/cortiq_engine/audiovae.rs
 *   [LTX] docs.rs cortiq-engine 0.6.3,  src/cortiq_engine/ltxaudio.rs
 *   [M3]  docs.rs cortiq-engine 0.5.89, src/cortiq_engine/music3.rs
 *
 * Layout everywhere: contiguous [B, C, T] float, T fastest.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_NOMEM 2

static inline double rnd(double v, int store_f64) {
    return store_f64 ? v : (double)(float)v;
}

/* ------------------------------------------------------------------ filter */

/* Modified Bessel function of the first kind, order 0, by its power series
 * sum_k ((x/2)^k / k!)^2.  [H3] `bessel_i0`: the term ratio is (x/2k)^2, the
 * loop stops once a term falls below 1e-18 of the sum, at most 39 terms. */
double orc_bessel_i0(double x) {
    double sum = 1.0, term = 1.0;
    for (int k = 1; k < 40; ++k) {
        double q = x / (2.0 * (double)k);
        term *= q * q;
        sum += term;
        if (term < 1e-18 * sum) break;
    }
    return sum;
}

/* sin(pi x)/(pi x), 1 at 0.  [H3] `sinc`. */
double orc_sinc(double x) {
    if (x == 0.0) return 1.0;
    return sin(M_PI * x) / (M_PI * x);
}

/* Kaiser-windowed sinc lowpass of `k` taps, normalised to unit sum.
 * [H3] `kaiser_sinc(cutoff, half_width, k)` (the reference's
 * kaiser_sinc_filter1d):
 *   half = k/2, delta_f = 4 half_width,
 *   A = 2.285 (half - 1) pi delta_f + 7.95  (Kaiser's attenuation estimate),
 *   beta = 0.1102 (A - 8.7) if A > 50, 0.5842 (A-21)^0.4 + 0.07886 (A-21)
 *          if 21 <= A <= 50, else 0,
 *   window_i = I0(beta sqrt(1 - r^2)) / I0(beta), r = 2i/(k-1) - 1,
 *   t_i = i - half + 0.5 for even k (half-integer sample points; the page
 *         gives only the even form, the odd form t_i = i - half is the
 *         natural centring and is not used by the decoder),
 *   tap_i = 2 cutoff window_i sinc(2 cutoff t_i), then divide by the sum.
 * Writes the double taps; the pages hand out float copies of them. */
int orc_kaiser_sinc(double cutoff, double half_width, int k, double *taps) {
    if (k <= 0 || !taps) return ORC_ERR_ARG;
    int half = k / 2;
    double delta_f = 4.0 * half_width;
    double A = 2.285 * ((double)half - 1.0) * M_PI * delta_f + 7.95;
    double beta;
    if (A > 50.0)
        beta = 0.1102 * (A - 8.7);
    else if (A >= 21.0)
        beta = 0.5842 * pow(A - 21.0, 0.4) + 0.07886 * (A - 21.0);
    else
        beta = 0.0;
    double denom = orc_bessel_i0(beta);
    double n = (double)k - 1.0;
    double sum = 0.0;
    for (int i = 0; i < k; ++i) {
        double r = (n > 0.0) ? 2.0 * (double)i / n - 1.0 : 0.0;
        double arg = 1.0 - r * r;
        if (arg < 0.0) arg = 0.0;
        double win = orc_bessel_i0(beta * sqrt(arg)) / denom;
        double t = (k % 2 == 0) ? -(double)half + (double)i + 0.5
                                : -(double)half + (double)i;
        taps[i] = 2.0 * cutoff * win * orc_sinc(2.0 * cutoff * t);
        sum += taps[i];
    }
    for (int i = 0; i < k; ++i) taps[i] /= sum;
    return ORC_OK;
}

/* --------------------------------------------------------------- activation */

static inline int clampi(long v, long lo, long hi) {
    return (int)(v < lo ? lo : (v > hi ? hi : v));
}

/* One channel row of the alias-free activation, in the pages' steps
 * ([H3] `Activation1d::apply`, `SnakeBeta::apply`, `fir_pad`;
 *  [LTX] `Aliasing::upsample`, `Aliasing::downsample`, `SnakeBeta::forward`):
 *  1. up: replicate-pad x by p = K/2 - 1 on both sides, transposed
 *     convolution at stride 2 with the up filter times the ratio 2,
 *     then trim p*2 + (K-2)/2 on the left and p*2 + ceil((K-2)/2) on the right;
 *  2. SnakeBeta on every up-sampled value: v += sin(a v)^2 * inv_b;
 *  3. down: replicate-pad by K/2 - 1 (even K) on the left and K/2 on the
 *     right, FIR with the down filter at stride 2.
 * `work` needs 2 * (2 n + 2 K + 8) doubles.  Returns the output length. */
static int act_row(const double *x, int n, double a, double inv_b,
                   const double *fu, const double *fd, int K, double *y,
                   double *work, int store_f64) {
    const int ratio = 2;
    int pad = K / ratio - 1;
    int pad_l = pad * ratio + (K - ratio) / 2;
    int pad_r = pad * ratio + (K - ratio + 1) / 2;
    int pn = n + 2 * pad;
    int full = (pn - 1) * ratio + K;
    double *up = work;
    for (int q = 0; q < full; ++q) up[q] = 0.0;
    for (int i = 0; i < pn; ++i) {
        double v = x[clampi((long)i - pad, 0, n - 1)] * (double)ratio;
        for (int j = 0; j < K; ++j) up[i * ratio + j] += v * fu[j];
    }
    int keep = full - pad_l - pad_r;
    double *mid = work + full;
    for (int m = 0; m < keep; ++m) {
        double u = rnd(up[pad_l + m], store_f64);  /* the page stores `up` */
        double s = sin(a * u);
        mid[m] = rnd(u + s * s * inv_b, store_f64);
    }
    int dpl = K / 2 - ((K % 2 == 0) ? 1 : 0);
    int dpr = K / 2;
    int padded = keep + dpl + dpr;
    int out_n = (padded - K) / ratio + 1;
    for (int t = 0; t < out_n; ++t) {
        double acc = 0.0;
        for (int j = 0; j < K; ++j)
            acc += fd[j] * mid[clampi((long)t * ratio + j - dpl, 0, keep - 1)];
        y[t] = rnd(acc, store_f64);
    }
    return out_n;
}

/* x, y: [rows, n] double; channel of row r is r % C. */
static void act_rows(const double *x, int rows, int C, int n,
                     const float *log_alpha, const float *log_beta,
                     const double *fu, const double *fd, int K, double eps,
                     double *y, double *work, int store_f64) {
    for (int r = 0; r < rows; ++r) {
        int c = r % C;
        /* [H3] exponentiates the stored logs at load; [LTX] per forward.
         * The oracle takes both exps in double. */
        double a = exp((double)log_alpha[c]);
        double inv_b = 1.0 / (exp((double)log_beta[c]) + eps);
        act_row(x + (size_t)r * n, n, a, inv_b, fu, fd, K, y + (size_t)r * n,
                work, store_f64);
    }
}

/* ------------------------------------------------------------------- convs */

/* Dilated Conv1d, zero padding:
 *   y[b,o,t] = bias[o] + sum_i sum_j w[o,i,j] x[b,i,t + j d - pad],
 *   Tout = T + 2 pad - d (K - 1).
 * [H3] `Conv1d::apply` (direct arm), [LTX] `Conv1d::forward` (im2col arm). */
static int conv_out_len(int T, int K, int d, int pad) {
    return T + 2 * pad - d * (K - 1);
}

static void conv1d_d(const double *x, int B, int Cin, int T, const float *w,
                     const float *bias, int Cout, int K, int d, int pad,
                     double *y, double *acc, int store_f64) {
    int Tout = conv_out_len(T, K, d, pad);
    for (int b = 0; b < B; ++b)
        for (int o = 0; o < Cout; ++o) {
            for (int t = 0; t < Tout; ++t) acc[t] = 0.0;
            for (int i = 0; i < Cin; ++i) {
                const double *xr = x + ((size_t)b * Cin + i) * T;
                for (int j = 0; j < K; ++j) {
                    double wv = (double)w[((size_t)o * Cin + i) * K + j];
                    long s = (long)j * d - pad;  /* input index = t + s */
                    long lo = s < 0 ? -s : 0;
                    long hi = (long)T - s;
                    if (hi > Tout) hi = Tout;
                    for (long t = lo; t < hi; ++t) acc[t] += wv * xr[t + s];
                }
            }
            double bo = bias ? (double)bias[o] : 0.0;
            double *yr = y + ((size_t)b * Cout + o) * Tout;
            for (int t = 0; t < Tout; ++t) yr[t] = rnd(acc[t] + bo, store_f64);
        }
}

/* ConvTranspose1d in the pages' scatter form:
 *   out[o, t s + j - pad] += x[i, t] w[i, o, j], kept where 0 <= . < Tout,
 *   Tout = (T - 1) s + K - 2 pad, bias added per output channel.
 * [H3] `ConvT1d::apply`, [LTX] `ConvT1d::forward`; weights [Cin, Cout, K]. */
static int convt_out_len(int T, int K, int s, int pad) {
    return (T - 1) * s + K - 2 * pad;
}

static void convt1d_d(const double *x, int B, int Cin, int T, const float *w,
                      const float *bias, int Cout, int K, int s, int pad,
                      double *y, double *acc, int store_f64) {
    int Tout = convt_out_len(T, K, s, pad);
    for (int b = 0; b < B; ++b)
        for (int o = 0; o < Cout; ++o) {
            for (int p = 0; p < Tout; ++p) acc[p] = 0.0;
            for (int i = 0; i < Cin; ++i) {
                const double *xr = x + ((size_t)b * Cin + i) * T;
                const float *wr = w + ((size_t)i * Cout + o) * K;
                for (int t = 0; t < T; ++t) {
                    double v = xr[t];
                    for (int j = 0; j < K; ++j) {
                        long p = (long)t * s + j - pad;
                        if (p >= 0 && p < Tout) acc[p] += v * (double)wr[j];
                    }
                }
            }
            double bo = bias ? (double)bias[o] : 0.0;
            double *yr = y + ((size_t)b * Cout + o) * Tout;
            for (int p = 0; p < Tout; ++p) yr[p] = rnd(acc[p] + bo, store_f64);
        }
}

static void final_op(double *y, size_t n, int final_act, int store_f64) {
    for (size_t i = 0; i < n; ++i) {
        double v = y[i];
        if (final_act == 1) v = v < -1.0 ? -1.0 : (v > 1.0 ? 1.0 : v);
        else if (final_act == 2) v = tanh(v);
        y[i] = rnd(v, store_f64);
    }
}

/* ------------------------------------------------------- exported wrappers */

static double *to_d(const float *x, size_t n) {
    double *d = (double *)malloc((n ? n : 1) * sizeof(double));
    if (!d) return NULL;
    for (size_t i = 0; i < n; ++i) d[i] = (double)x[i];
    return d;
}

static void to_f(const double *d, float *y, size_t n) {
    for (size_t i = 0; i < n; ++i) y[i] = (float)d[i];
}

static int up_filter_ok(int K) { return K >= 2 && K % 2 == 0; }

/* Alias-free activation over [B, C, T]; filters are K float taps each. */
int orc_activation1d(const float *x, int B, int C, int T,
                     const float *log_alpha, const float *log_beta,
                     const float *up, const float *down, int K, double eps,
                     int store_f64, float *y) {
    if (B < 0 || C <= 0 || T <= 0 || !up_filter_ok(K)) return ORC_ERR_ARG;
    size_t n = (size_t)B * C * T;
    double fu[64], fd[64];
    if (K > 64) return ORC_ERR_ARG;
    for (int j = 0; j < K; ++j) { fu[j] = up[j]; fd[j] = down[j]; }
    double *xd = to_d(x, n), *yd = (double *)malloc((n ? n : 1) * sizeof(double));
    double *work = (double *)malloc((size_t)2 * (2 * T + 2 * K + 8) * sizeof(double));
    if (!xd || !yd || !work) { free(xd); free(yd); free(work); return ORC_ERR_NOMEM; }
    act_rows(xd, B * C, C, T, log_alpha, log_beta, fu, fd, K, eps, yd, work, store_f64);
    to_f(yd, y, n);
    free(xd); free(yd); free(work);
    return ORC_OK;
}

int orc_conv1d(const float *x, int B, int Cin, int T, const float *w,
               const float *bias, int Cout, int K, int d, int pad,
               int store_f64, float *y) {
    int Tout = conv_out_len(T, K, d, pad);
    if (B < 0 || Cin <= 0 || Cout <= 0 || K <= 0 || d <= 0 || pad < 0 || Tout <= 0)
        return ORC_ERR_ARG;
    size_t nin = (size_t)B * Cin * T, nout = (size_t)B * Cout * Tout;
    double *xd = to_d(x, nin), *yd = (double *)malloc((nout ? nout : 1) * sizeof(double));
    double *acc = (double *)malloc((size_t)Tout * sizeof(double));
    if (!xd || !yd || !acc) { free(xd); free(yd); free(acc); return ORC_ERR_NOMEM; }
    conv1d_d(xd, B, Cin, T, w, bias, Cout, K, d, pad, yd, acc, store_f64);
    to_f(yd, y, nout);
    free(xd); free(yd); free(acc);
    return ORC_OK;
}

/* The latent front end of [H3] `AudioVae::decode`.  The normalised latents
 * arrive as z [C, S, T] (channel ci of side s at (ci S + s) T + t; the page's
 * stereo layout has S = 2).  Per side s, in the page's order:
 *   lat[ci, t] = z[ci, s, t] std[ci] + mean[ci]      (stored as float),
 *   out[s, o, t] = bias[o] + sum_ci w[o, ci] lat[ci, t]   (`dec_in`).
 * `dec_in` is the checkpoint's `avae.dec_in_proj` Conv1d, loaded with padding
 * 0 and dilation 1 ([H3] `AudioVae::from_cmf`); `decode` keeps the length t
 * after it, so its kernel has one tap: w [Cout, C, 1]. */
int orc_latent_front_end(const float *z, int C, int S, int T, const float *mean,
                         const float *std_, const float *w, const float *bias,
                         int Cout, int store_f64, float *out) {
    if (C <= 0 || S <= 0 || T <= 0 || Cout <= 0 || !mean || !std_ || !w) return ORC_ERR_ARG;
    size_t nl = (size_t)S * C * T, no = (size_t)S * Cout * T;
    double *lat = (double *)malloc(nl * sizeof(double));
    double *yd = (double *)malloc(no * sizeof(double));
    double *acc = (double *)malloc((size_t)T * sizeof(double));
    if (!lat || !yd || !acc) { free(lat); free(yd); free(acc); return ORC_ERR_NOMEM; }
    for (int s = 0; s < S; ++s)
        for (int ci = 0; ci < C; ++ci) {
            const float *zr = z + ((size_t)ci * S + s) * T;
            double *lr = lat + ((size_t)s * C + ci) * T;
            for (int t = 0; t < T; ++t)
                lr[t] = rnd((double)zr[t] * (double)std_[ci] + (double)mean[ci], store_f64);
        }
    conv1d_d(lat, S, C, T, w, bias, Cout, 1, 1, 0, yd, acc, store_f64);
    to_f(yd, out, no);
    free(lat); free(yd); free(acc);
    return ORC_OK;
}

int orc_conv_transpose1d(const float *x, int B, int Cin, int T, const float *w,
                         const float *bias, int Cout, int K, int s, int pad,
                         int store_f64, float *y) {
    if (B < 0 || Cin <= 0 || Cout <= 0 || K <= 0 || s <= 0 || pad < 0 || T <= 0)
        return ORC_ERR_ARG;
    int Tout = convt_out_len(T, K, s, pad);
    if (Tout <= 0) return ORC_ERR_ARG;
    size_t nin = (size_t)B * Cin * T, nout = (size_t)B * Cout * Tout;
    double *xd = to_d(x, nin), *yd = (double *)malloc((nout ? nout : 1) * sizeof(double));
    double *acc = (double *)malloc((size_t)Tout * sizeof(double));
    if (!xd || !yd || !acc) { free(xd); free(yd); free(acc); return ORC_ERR_NOMEM; }
    convt1d_d(xd, B, Cin, T, w, bias, Cout, K, s, pad, yd, acc, store_f64);
    to_f(yd, y, nout);
    free(xd); free(yd); free(acc);
    return ORC_OK;
}

/* Single output points of the three layer kinds, for spot checks of large
 * tensors.  `idx` holds n_pts triples (b, c, t); the result is the layer's
 * output at each point (before any rounding).  Same definitions as above. */
int orc_conv1d_points(const float *x, int B, int Cin, int T, const float *w,
                      const float *bias, int Cout, int K, int d, int pad,
                      const int64_t *idx, int n_pts, double *out) {
    int Tout = conv_out_len(T, K, d, pad);
    for (int q = 0; q < n_pts; ++q) {
        long b = idx[3 * q], o = idx[3 * q + 1], t = idx[3 * q + 2];
        if (b < 0 || b >= B || o < 0 || o >= Cout || t < 0 || t >= Tout) return ORC_ERR_ARG;
        double acc = 0.0;
        for (int i = 0; i < Cin; ++i)
            for (int j = 0; j < K; ++j) {
                long p = t + (long)j * d - pad;
                if (p >= 0 && p < T)
                    acc += (double)w[((size_t)o * Cin + i) * K + j] *
                           (double)x[((size_t)b * Cin + i) * T + p];
            }
        out[q] = acc + (bias ? (double)bias[o] : 0.0);
    }
    return ORC_OK;
}

int orc_conv_transpose1d_points(const float *x, int B, int Cin, int T,
                                const float *w, const float *bias, int Cout,
                                int K, int s, int pad, const int64_t *idx,
                                int n_pts, double *out) {
    int Tout = convt_out_len(T, K, s, pad);
    for (int q = 0; q < n_pts; ++q) {
        long b = idx[3 * q], o = idx[3 * q + 1], p = idx[3 * q + 2];
        if (b < 0 || b >= B || o < 0 || o >= Cout || p < 0 || p >= Tout) return ORC_ERR_ARG;
        double acc = 0.0;
        /* every (t, j) whose scatter target t s + j - pad is p */
        for (int i = 0; i < Cin; ++i)
            for (int t = 0; t < T; ++t)
                for (int j = 0; j < K; ++j)
                    if ((long)t * s + j - pad == p)
                        acc += (double)x[((size_t)b * Cin + i) * T + t] *
                               (double)w[((size_t)i * Cout + o) * K + j];
        out[q] = acc + (bias ? (double)bias[o] : 0.0);
    }
    return ORC_OK;
}

int orc_activation1d_points(const float *x, int B, int C, int T,
                            const float *log_alpha, const float *log_beta,
                            const float *up, const float *down, int K,
                            double eps, const int64_t *idx, int n_pts,
                            double *out) {
    if (!up_filter_ok(K) || K > 64) return ORC_ERR_ARG;
    double fu[64], fd[64];
    for (int j = 0; j < K; ++j) { fu[j] = up[j]; fd[j] = down[j]; }
    /* the activation is local: output t depends on inputs within K of t, so
     * run the row definition on a window that is exact at t (the window is
     * the whole row when the row is short). */
    int W = 8 * K;
    double *xw = (double *)malloc((size_t)(2 * W + 1) * sizeof(double));
    double *yw = (double *)malloc((size_t)(2 * W + 1) * sizeof(double));
    double *work = (double *)malloc((size_t)2 * (2 * (2 * W + 1) + 2 * K + 8) * sizeof(double));
    if (!xw || !yw || !work) { free(xw); free(yw); free(work); return ORC_ERR_NOMEM; }
    for (int q = 0; q < n_pts; ++q) {
        long b = idx[3 * q], c = idx[3 * q + 1], t = idx[3 * q + 2];
        if (b < 0 || b >= B || c < 0 || c >= C || t < 0 || t >= T) {
            free(xw); free(yw); free(work);
            return ORC_ERR_ARG;
        }
        /* window [lo, hi) of the row; where it is cut short of the row's end,
         * the cut sits W samples from t, far outside t's support. */
        long lo = t - W < 0 ? 0 : t - W;
        long hi = t + W + 1 > T ? T : t + W + 1;
        const float *xr = x + ((size_t)b * C + c) * T;
        for (long p = lo; p < hi; ++p) xw[p - lo] = (double)xr[p];
        double a = exp((double)log_alpha[c]);
        double inv_b = 1.0 / (exp((double)log_beta[c]) + eps);
        act_row(xw, (int)(hi - lo), a, inv_b, fu, fd, K, yw, work, 1);
        out[q] = yw[t - lo];
    }
    free(xw); free(yw); free(work);
    return ORC_OK;
}

/* ----------------------------------------------------------------- decoder */

/* Decoder geometry, as an int array (the oracle's own description):
 *  [0] in_ch   [1] pre_ch  [2] pre_k  [3] n_up
 *  [4..11]  up_rate[8]   [12..19] up_k[8]   [20..27] up_ch[8]
 *  [28] n_blocks  [29..32] block_k[4]  [33] n_dil  [34..37] dil[4]
 *  [38] post_k  [39] out_ch  [40] final_act (0 none, 1 clamp, 2 tanh)
 * Parameter order in the flat `params` array (module order):
 *  conv_pre w [pre_ch, in_ch, pre_k], b [pre_ch];
 *  per stage i: ups w [Cin_i, Cout_i, up_k_i], b [Cout_i];
 *    per block j, per dilation u: act1 log_alpha [C], log_beta [C],
 *      conv1 w [C, C, K_j], b [C], act2 log_alpha [C], log_beta [C],
 *      conv2 w [C, C, K_j], b [C];
 *  act_post log_alpha [C], log_beta [C]; conv_post w [out, C, post_k], b [out].
 * Stage wiring [H3] `AudioVae::from_cmf` / `decode`, [LTX] `Vocoder`:
 *  conv_pre (pad (k-1)/2) -> per stage ConvT (pad (k - s)/2), then the mean
 *  of the stage's AMP blocks, each block a chain of residual units
 *  cur += conv2(act2(conv1(act1(cur)))) with conv1 dilated
 *  (pad (K d - d)/2) and conv2 undilated -> act_post -> conv_post
 *  (pad (k-1)/2) -> final op. */
enum { G_IN, G_PRE_CH, G_PRE_K, G_NUP, G_RATE = 4, G_UPK = 12, G_UPCH = 20,
       G_NB = 28, G_BK = 29, G_ND = 33, G_DIL = 34, G_POSTK = 38, G_OUT = 39,
       G_FINAL = 40, G_LEN = 41 };

static int geo_ok(const int *g) {
    if (g[G_IN] <= 0 || g[G_PRE_CH] <= 0 || g[G_PRE_K] <= 0) return 0;
    if (g[G_NUP] < 0 || g[G_NUP] > 8) return 0;
    if (g[G_NB] < 1 || g[G_NB] > 4 || g[G_ND] < 1 || g[G_ND] > 4) return 0;
    for (int i = 0; i < g[G_NUP]; ++i)
        if (g[G_RATE + i] <= 0 || g[G_UPK + i] < g[G_RATE + i] || g[G_UPCH + i] <= 0) return 0;
    for (int j = 0; j < g[G_NB]; ++j) if (g[G_BK + j] <= 0 || g[G_BK + j] % 2 == 0) return 0;
    for (int u = 0; u < g[G_ND]; ++u) if (g[G_DIL + u] <= 0) return 0;
    if (g[G_POSTK] <= 0 || g[G_POSTK] % 2 == 0 || g[G_PRE_K] % 2 == 0) return 0;
    if (g[G_OUT] <= 0) return 0;
    return 1;
}

long orc_decoder_param_count(const int *g) {
    if (!geo_ok(g)) return -1;
    long n = 0;
    long cin = g[G_PRE_CH];
    n += (long)g[G_PRE_CH] * g[G_IN] * g[G_PRE_K] + g[G_PRE_CH];
    for (int i = 0; i < g[G_NUP]; ++i) {
        long c = g[G_UPCH + i];
        n += cin * c * g[G_UPK + i] + c;
        for (int j = 0; j < g[G_NB]; ++j)
            n += (long)g[G_ND] * (4 * c + 2 * (c * c * g[G_BK + j] + c));
        cin = c;
    }
    n += 2 * cin + (long)g[G_OUT] * cin * g[G_POSTK] + g[G_OUT];
    return n;
}

/* Samples per latent frame (product of the rates). */
long orc_decoder_hop(const int *g) {
    long h = 1;
    for (int i = 0; i < g[G_NUP]; ++i) h *= g[G_RATE + i];
    return h;
}

/* Full-rate length before the final trim, from `frames` latent frames. */
static long layer_len(const int *g, long frames) {
    long n = frames;  /* conv_pre keeps the length (odd k, pad (k-1)/2) */
    for (int i = 0; i < g[G_NUP]; ++i) {
        int s = g[G_RATE + i], k = g[G_UPK + i];
        n = (n - 1) * s + k - 2 * ((k - s) / 2);
    }
    return n;
}

long orc_decoder_raw_len(const int *g, int frames) { return layer_len(g, frames); }

/* One AMP block on cur [B, C, n] (in place).  [H3] `AmpBlock::apply`,
 * [LTX] `AmpBlock::forward`. */
static const float *amp_block(double *cur, int B, int C, int n, int K,
                              const int *dil, int nd, const float *p,
                              const double *fu, const double *fd, int FK,
                              double eps, double *h1, double *h2, double *acc,
                              double *work, int store_f64) {
    size_t cw = (size_t)C * C * K;
    for (int u = 0; u < nd; ++u) {
        const float *a1a = p; p += C;
        const float *a1b = p; p += C;
        const float *c1w = p; p += cw;
        const float *c1b = p; p += C;
        const float *a2a = p; p += C;
        const float *a2b = p; p += C;
        const float *c2w = p; p += cw;
        const float *c2b = p; p += C;
        int d = dil[u];
        act_rows(cur, B * C, C, n, a1a, a1b, fu, fd, FK, eps, h1, work, store_f64);
        conv1d_d(h1, B, C, n, c1w, c1b, C, K, d, (K * d - d) / 2, h2, acc, store_f64);
        act_rows(h2, B * C, C, n, a2a, a2b, fu, fd, FK, eps, h1, work, store_f64);
        conv1d_d(h1, B, C, n, c2w, c2b, C, K, 1, (K - 1) / 2, h2, acc, store_f64);
        size_t tot = (size_t)B * C * n;
        for (size_t q = 0; q < tot; ++q) cur[q] = rnd(cur[q] + h2[q], store_f64);
    }
    return p;
}

/* One AMP block on x [B, C, T] -> y, parameters in the block's module order
 * (per dilation: act1 log_alpha, log_beta, conv1 w, b, act2 log_alpha,
 * log_beta, conv2 w, b).  Same definition as inside the decoder. */
int orc_amp_block(const float *x, int B, int C, int T, const float *params, int K,
                  const int *dil, int nd, const float *up, const float *down, int FK,
                  double eps, int store_f64, float *y) {
    if (B <= 0 || C <= 0 || T <= 0 || K <= 0 || K % 2 == 0 || nd <= 0 || nd > 4 ||
        !up_filter_ok(FK) || FK > 64)
        return ORC_ERR_ARG;
    for (int u = 0; u < nd; ++u) if (dil[u] <= 0) return ORC_ERR_ARG;
    double fu[64], fd[64];
    for (int j = 0; j < FK; ++j) { fu[j] = up[j]; fd[j] = down[j]; }
    size_t n = (size_t)B * C * T;
    double *cur = to_d(x, n);
    double *h1 = (double *)malloc(n * sizeof(double));
    double *h2 = (double *)malloc(n * sizeof(double));
    double *acc = (double *)malloc((size_t)(T + 8) * sizeof(double));
    double *work = (double *)malloc((size_t)2 * (2 * T + 2 * FK + 8) * sizeof(double));
    if (!cur || !h1 || !h2 || !acc || !work) {
        free(cur); free(h1); free(h2); free(acc); free(work);
        return ORC_ERR_NOMEM;
    }
    amp_block(cur, B, C, T, K, dil, nd, params, fu, fd, FK, eps, h1, h2, acc, work, store_f64);
    to_f(cur, y, n);
    free(cur); free(h1); free(h2); free(acc); free(work);
    return ORC_OK;
}

/* Decode z [B, in_ch, frames] -> y [B, out_ch, frames * hop] (the first
 * frames*hop samples of the full-rate signal; the pages' odd-stride ConvT
 * makes the raw signal a few samples longer, and the extra samples sit at
 * the end).  `up`/`down` are the activation filters (FK taps). */
int orc_decode(const int *g, const float *params, const float *z, int B,
               int frames, const float *up, const float *down, int FK,
               double eps, int store_f64, float *y) {
    if (!geo_ok(g) || B <= 0 || frames <= 0 || !up_filter_ok(FK) || FK > 64)
        return ORC_ERR_ARG;
    double fu[64], fd[64];
    for (int j = 0; j < FK; ++j) { fu[j] = up[j]; fd[j] = down[j]; }
    /* largest B*C*n over the layers, and the longest row */
    long n = frames, maxel = (long)B * g[G_IN] * frames, maxn = frames;
    if ((long)B * g[G_PRE_CH] * n > maxel) maxel = (long)B * g[G_PRE_CH] * n;
    for (int i = 0; i < g[G_NUP]; ++i) {
        int s = g[G_RATE + i], k = g[G_UPK + i];
        n = (n - 1) * s + k - 2 * ((k - s) / 2);
        if ((long)B * g[G_UPCH + i] * n > maxel) maxel = (long)B * g[G_UPCH + i] * n;
        if (n > maxn) maxn = n;
    }
    if ((long)B * g[G_OUT] * n > maxel) maxel = (long)B * g[G_OUT] * n;
    long raw = n;
    size_t E = (size_t)maxel;
    double *x = (double *)malloc(E * sizeof(double));
    double *st = (double *)malloc(E * sizeof(double));
    double *cur = (double *)malloc(E * sizeof(double));
    double *h1 = (double *)malloc(E * sizeof(double));
    double *h2 = (double *)malloc(E * sizeof(double));
    double *acc = (double *)malloc((size_t)(maxn + 8) * sizeof(double));
    double *work = (double *)malloc((size_t)2 * (2 * maxn + 2 * FK + 8) * sizeof(double));
    if (!x || !st || !cur || !h1 || !h2 || !acc || !work) {
        free(x); free(st); free(cur); free(h1); free(h2); free(acc); free(work);
        return ORC_ERR_NOMEM;
    }
    const float *p = params;
    /* latent, then conv_pre */
    size_t nz = (size_t)B * g[G_IN] * frames;
    for (size_t q = 0; q < nz; ++q) h1[q] = (double)z[q];
    int C = g[G_PRE_CH];
    const float *pw = p; p += (size_t)C * g[G_IN] * g[G_PRE_K];
    const float *pb = p; p += C;
    conv1d_d(h1, B, g[G_IN], frames, pw, pb, C, g[G_PRE_K], 1, (g[G_PRE_K] - 1) / 2,
             x, acc, store_f64);
    n = frames;
    for (int i = 0; i < g[G_NUP]; ++i) {
        int s = g[G_RATE + i], k = g[G_UPK + i], Co = g[G_UPCH + i];
        const float *uw = p; p += (size_t)C * Co * k;
        const float *ub = p; p += Co;
        int pad = (k - s) / 2;
        int n2 = convt_out_len((int)n, k, s, pad);
        convt1d_d(x, B, C, (int)n, uw, ub, Co, k, s, pad, h1, acc, store_f64);
        C = Co;
        n = n2;
        size_t tot = (size_t)B * C * n;
        memcpy(x, h1, tot * sizeof(double));  /* x = stage input */
        for (size_t q = 0; q < tot; ++q) st[q] = 0.0;
        for (int j = 0; j < g[G_NB]; ++j) {
            memcpy(cur, x, tot * sizeof(double));
            p = amp_block(cur, B, C, (int)n, g[G_BK + j], g + G_DIL, g[G_ND], p, fu,
                          fd, FK, eps, h1, h2, acc, work, store_f64);
            for (size_t q = 0; q < tot; ++q) st[q] = rnd(st[q] + cur[q], store_f64);
        }
        /* the mean of the blocks: the pages sum them, then scale by 1/nb */
        double inv = store_f64 ? 1.0 / (double)g[G_NB] : (double)(1.0f / (float)g[G_NB]);
        for (size_t q = 0; q < tot; ++q) x[q] = rnd(st[q] * inv, store_f64);
    }
    const float *la = p; p += C;
    const float *lb = p; p += C;
    act_rows(x, B * C, C, (int)n, la, lb, fu, fd, FK, eps, h1, work, store_f64);
    const float *ow = p; p += (size_t)g[G_OUT] * C * g[G_POSTK];
    const float *ob = p; p += g[G_OUT];
    conv1d_d(h1, B, C, (int)n, ow, ob, g[G_OUT], g[G_POSTK], 1, (g[G_POSTK] - 1) / 2,
             h2, acc, store_f64);
    final_op(h2, (size_t)B * g[G_OUT] * n, g[G_FINAL], store_f64);
    long hop = orc_decoder_hop(g);
    long L = (long)frames * hop;
    if (L > raw) L = raw;
    for (int b = 0; b < B; ++b)
        for (int o = 0; o < g[G_OUT]; ++o)
            for (long t = 0; t < L; ++t)
                y[((size_t)b * g[G_OUT] + o) * L + t] =
                    (float)h2[((size_t)b * g[G_OUT] + o) * raw + t];
    free(x); free(st); free(cur); free(h1); free(h2); free(acc); free(work);
    return ORC_OK;
}

/* Time-tiled decode.  Tiles of `tile` frames start every tile - overlap
 * frames; the last tile is cut at `frames`, and the loop stops with the tile
 * that reaches the end.  Each tile is decoded on its own (its own edges are
 * padded as a whole signal's would be), and where tiles overlap the samples
 * are averaged by the number of tiles covering them -- the windowing rule of
 * [M3] `Music3Dit::forward_windowed`.  `tile_lo`..`tile_hi` (exclusive) picks
 * which tiles contribute; samples no picked tile covers are left as NaN and
 * `count` gets the per-sample coverage (may be NULL). */
int orc_decode_tiled(const int *g, const float *params, const float *z, int B,
                     int frames, int tile, int overlap, int tile_lo,
                     int tile_hi, const float *up, const float *down, int FK,
                     double eps, int store_f64, float *y, float *count) {
    if (!geo_ok(g) || tile <= 0 || overlap < 0 || overlap >= tile) return ORC_ERR_ARG;
    long hop = orc_decoder_hop(g);
    int O = g[G_OUT];
    long L = (long)frames * hop;
    double *sum = (double *)calloc((size_t)B * O * L, sizeof(double));
    double *cnt = (double *)calloc((size_t)L, sizeof(double));
    if (!sum || !cnt) { free(sum); free(cnt); return ORC_ERR_NOMEM; }
    int start = 0, ti = 0, rc = ORC_OK;
    for (;;) {
        int len = frames - start < tile ? frames - start : tile;
        if (ti >= tile_lo && ti < tile_hi) {
            float *zt = (float *)malloc((size_t)B * g[G_IN] * len * sizeof(float));
            float *yt = (float *)malloc((size_t)B * O * len * hop * sizeof(float));
            if (!zt || !yt) { free(zt); free(yt); rc = ORC_ERR_NOMEM; break; }
            for (int b = 0; b < B; ++b)
                for (int c = 0; c < g[G_IN]; ++c)
                    memcpy(zt + ((size_t)b * g[G_IN] + c) * len,
                           z + ((size_t)b * g[G_IN] + c) * frames + start,
                           (size_t)len * sizeof(float));
            rc = orc_decode(g, params, zt, B, len, up, down, FK, eps, store_f64, yt);
            if (rc == ORC_OK) {
                long tl = (long)len * hop, off = (long)start * hop;
                for (int b = 0; b < B; ++b)
                    for (int o = 0; o < O; ++o)
                        for (long t = 0; t < tl; ++t)
                            sum[((size_t)b * O + o) * L + off + t] +=
                                (double)yt[((size_t)b * O + o) * tl + t];
                for (long t = 0; t < tl; ++t) cnt[off + t] += 1.0;
            }
            free(zt); free(yt);
            if (rc != ORC_OK) break;
        }
        if (start + len >= frames) break;
        start += tile - overlap;
        ++ti;
    }
    if (rc == ORC_OK) {
        for (int b = 0; b < B; ++b)
            for (int o = 0; o < O; ++o)
                for (long t = 0; t < L; ++t) {
                    double c = cnt[t];
                    y[((size_t)b * O + o) * L + t] =
                        c > 0.0 ? (float)(sum[((size_t)b * O + o) * L + t] / c) : (float)NAN;
                }
        if (count)
            for (long t = 0; t < L; ++t) count[t] = (float)cnt[t];
    }
    free(sum); free(cnt);
    return rc;
}

/* Number of tiles the tiling rule above produces. */
int orc_tile_count(int frames, int tile, int overlap) {
    if (frames <= 0 || tile <= 0 || overlap < 0 || overlap >= tile) return -1;
    int start = 0, n = 1;
    while (start + tile < frames) { start += tile - overlap; ++n; }
    return n;
}

/* ------------------------------------------------------ Music-3 DAV decoder */

/* Plain Snake over rows of length n, alpha used as stored ([H3] `Snake`):
 *   v = x + sin^2(alpha_c x) / (alpha_c + 1e-9). */
static void snake_rows(double *x, int rows, int C, int n, const float *alpha,
                       int store_f64) {
    for (int r = 0; r < rows; ++r) {
        double a = (double)alpha[r % C];
        double inv = 1.0 / (a + 1e-9);
        double *xr = x + (size_t)r * n;
        for (int t = 0; t < n; ++t) {
            double s = sin(a * xr[t]);
            xr[t] = rnd(xr[t] + s * s * inv, store_f64);
        }
    }
}

/* Plain Snake over x [B, C, T] (exported for its pins). */
int orc_snake1d(const float *x, int B, int C, int T, const float *alpha, int store_f64,
                float *y) {
    if (B <= 0 || C <= 0 || T <= 0 || !alpha) return ORC_ERR_ARG;
    size_t n = (size_t)B * C * T;
    double *d = to_d(x, n);
    if (!d) return ORC_ERR_NOMEM;
    snake_rows(d, B * C, C, T, alpha, store_f64);
    to_f(d, y, n);
    free(d);
    return ORC_OK;
}

/* DAV geometry, as an int array:
 *  [0] latent_ch  [1] in_ch (dec_in output)  [2] pre_ch  [3] pre_k  [4] n_up
 *  [5..12] up_rate[8]  [13..20] up_k[8]  [21..28] up_ch[8]
 *  [29] n_dil  [30..33] dil[4]  [34] unit_k  [35] post_k  [36] out_ch
 *  [37] final_act (0 none, 1 clamp, 2 tanh).
 * Parameters in module order ([H3] `Music3Dav::from_cmf`, `DavStage::load`,
 * `DavUnit::load`): dec_in w [in, lat, 1], b [in]; conv_pre w [pre, in,
 * pre_k], b [pre]; per stage i: act alpha [Cin_i]; up w [Cin_i, Cout_i,
 * up_k_i], b [Cout_i]; per unit u: a1 alpha [C], c1 w [C, C, unit_k], b [C],
 * a2 alpha [C], c2 w [C, C, 1], b [C]; act_post alpha [C]; conv_post w [out,
 * C, post_k], b [out].
 * Wiring ([H3] `Music3Dav::decode`, `DavStage::apply`, `DavUnit::apply`):
 *  dec_in (one tap, pad 0) -> conv_pre (pad (k-1)/2) -> per stage: Snake ->
 *  ConvT (pad (k - s)/2) -> units x += c2(Snake(c1(Snake(x)))) with c1
 *  dilated (pad d (unit_k - 1)/2) and c2 one tap -> Snake -> conv_post
 *  (pad (k-1)/2) -> final op. */
enum { D_LAT, D_IN, D_PRE, D_PREK, D_NUP, D_RATE = 5, D_UPK = 13, D_UPCH = 21,
       D_ND = 29, D_DIL = 30, D_UNITK = 34, D_POSTK = 35, D_OUT = 36, D_FINAL = 37,
       D_LEN = 38 };

static int dav_ok(const int *g) {
    if (g[D_LAT] <= 0 || g[D_IN] <= 0 || g[D_PRE] <= 0 || g[D_PREK] <= 0 ||
        g[D_PREK] % 2 == 0) return 0;
    if (g[D_NUP] < 0 || g[D_NUP] > 8 || g[D_ND] < 0 || g[D_ND] > 4) return 0;
    for (int i = 0; i < g[D_NUP]; ++i)
        if (g[D_RATE + i] <= 0 || g[D_UPK + i] < g[D_RATE + i] || g[D_UPCH + i] <= 0) return 0;
    for (int u = 0; u < g[D_ND]; ++u) if (g[D_DIL + u] <= 0) return 0;
    if (g[D_UNITK] <= 0 || g[D_UNITK] % 2 == 0 || g[D_POSTK] <= 0 || g[D_POSTK] % 2 == 0)
        return 0;
    return g[D_OUT] > 0;
}

long orc_dav_param_count(const int *g) {
    if (!dav_ok(g)) return -1;
    long n = (long)g[D_IN] * g[D_LAT] + g[D_IN];
    n += (long)g[D_PRE] * g[D_IN] * g[D_PREK] + g[D_PRE];
    long cin = g[D_PRE];
    for (int i = 0; i < g[D_NUP]; ++i) {
        long c = g[D_UPCH + i];
        n += cin + cin * c * g[D_UPK + i] + c;
        n += (long)g[D_ND] * (2 * c + c * c * g[D_UNITK] + c + c * c + c);
        cin = c;
    }
    n += cin + (long)g[D_OUT] * cin * g[D_POSTK] + g[D_OUT];
    return n;
}

long orc_dav_hop(const int *g) {
    long h = 1;
    for (int i = 0; i < g[D_NUP]; ++i) h *= g[D_RATE + i];
    return h;
}

/* z [B, lat, F] -> y [B, out, F hop].  Every ConvT must give exactly s times
 * its input length (k - 2 pad = s), as the page's `n = n * stride` assumes;
 * otherwise ORC_ERR_ARG. */
int orc_dav_decode(const int *g, const float *params, const float *z, int B, int F,
                   int store_f64, float *y) {
    if (!dav_ok(g) || B <= 0 || F <= 0) return ORC_ERR_ARG;
    long hop = orc_dav_hop(g);
    long L = (long)F * hop;
    int cmax = g[D_PRE] > g[D_IN] ? g[D_PRE] : g[D_IN];
    if (g[D_LAT] > cmax) cmax = g[D_LAT];
    for (int i = 0; i < g[D_NUP]; ++i) {
        int k = g[D_UPK + i], s = g[D_RATE + i];
        if (k - 2 * ((k - s) / 2) != s) return ORC_ERR_ARG;
        if (g[D_UPCH + i] > cmax) cmax = g[D_UPCH + i];
    }
    size_t big = (size_t)B * cmax * (size_t)L + 16;
    double *a = (double *)malloc(big * sizeof(double));
    double *b = (double *)malloc(big * sizeof(double));
    double *r = (double *)malloc(big * sizeof(double));
    double *acc = (double *)malloc(((size_t)L + 64) * sizeof(double));
    if (!a || !b || !r || !acc) { free(a); free(b); free(r); free(acc); return ORC_ERR_NOMEM; }
    const float *p = params;
    size_t nz = (size_t)B * g[D_LAT] * F;
    for (size_t i = 0; i < nz; ++i) a[i] = (double)z[i];
    /* dec_in */
    const float *w = p; p += (size_t)g[D_IN] * g[D_LAT];
    const float *bb = p; p += g[D_IN];
    conv1d_d(a, B, g[D_LAT], F, w, bb, g[D_IN], 1, 1, 0, b, acc, store_f64);
    /* conv_pre */
    w = p; p += (size_t)g[D_PRE] * g[D_IN] * g[D_PREK];
    bb = p; p += g[D_PRE];
    conv1d_d(b, B, g[D_IN], F, w, bb, g[D_PRE], g[D_PREK], 1, (g[D_PREK] - 1) / 2, a, acc,
             store_f64);
    int C = g[D_PRE];
    long n = F;
    for (int i = 0; i < g[D_NUP]; ++i) {
        int s = g[D_RATE + i], k = g[D_UPK + i], Co = g[D_UPCH + i];
        const float *alpha = p; p += C;
        snake_rows(a, B * C, C, (int)n, alpha, store_f64);
        w = p; p += (size_t)C * Co * k;
        bb = p; p += Co;
        convt1d_d(a, B, C, (int)n, w, bb, Co, k, s, (k - s) / 2, b, acc, store_f64);
        n *= s;
        C = Co;
        size_t nn = (size_t)B * C * n;
        for (int u = 0; u < g[D_ND]; ++u) {
            int d = g[D_DIL + u], K = g[D_UNITK];
            const float *a1 = p; p += C;
            const float *w1 = p; p += (size_t)C * C * K;
            const float *b1 = p; p += C;
            const float *a2 = p; p += C;
            const float *w2 = p; p += (size_t)C * C;
            const float *b2 = p; p += C;
            memcpy(r, b, nn * sizeof(double));
            snake_rows(r, B * C, C, (int)n, a1, store_f64);
            conv1d_d(r, B, C, (int)n, w1, b1, C, K, d, d * (K - 1) / 2, a, acc, store_f64);
            snake_rows(a, B * C, C, (int)n, a2, store_f64);
            conv1d_d(a, B, C, (int)n, w2, b2, C, 1, 1, 0, r, acc, store_f64);
            for (size_t q = 0; q < nn; ++q) b[q] = rnd(b[q] + r[q], store_f64);
        }
        /* the stage output lives in b; the next stage reads a */
        memcpy(a, b, nn * sizeof(double));
    }
    const float *ap = p; p += C;
    snake_rows(a, B * C, C, (int)n, ap, store_f64);
    w = p; p += (size_t)g[D_OUT] * C * g[D_POSTK];
    bb = p; p += g[D_OUT];
    conv1d_d(a, B, C, (int)n, w, bb, g[D_OUT], g[D_POSTK], 1, (g[D_POSTK] - 1) / 2, b, acc,
             store_f64);
    size_t ny = (size_t)B * g[D_OUT] * L;
    final_op(b, ny, g[D_FINAL], store_f64);
    to_f(b, y, ny);
    free(a); free(b); free(r); free(acc);
    return ORC_OK;
}

/* ------------------------------------------- LTX bandwidth-extension tail */

/* The causal log-mel the bandwidth extender is conditioned on ([LTX]
 * `MelStft::forward`): the signal x [C, T] is left-padded with
 * L - hop zeros, frame f starts at f hop, frames = (T + L - hop - L)/hop + 1,
 *   re[r] = sum_j v[j] basis[r, j],  im[r] = sum_j v[j] basis[n_freqs + r, j],
 *   mag[r] = sqrt(re^2 + im^2)                       (stored as float),
 *   mel[m] = ln(max(sum_r mel_basis[m, r] mag[r], 1e-5)),
 * written in the generator's folded layout out[c n_mels + m, f] ([LTX]
 * `Vocoder::forward` folds (channel, mel) into one channel axis).
 * basis [2 n_freqs, L] (DFT x window rows), mel_basis [n_mels, n_freqs]. */
int orc_mel_stft(const float *x, int C, int T, const float *basis, int n_freqs, int L,
                 int hop, const float *mel_basis, int n_mels, int store_f64, float *out) {
    if (C <= 0 || T <= 0 || n_freqs <= 0 || L <= 0 || hop <= 0 || n_mels <= 0) return ORC_ERR_ARG;
    long left = L > hop ? L - hop : 0;
    long padded = T + left;
    if (padded < L) return ORC_ERR_ARG;
    long frames = (padded - L) / hop + 1;
    double *mag = (double *)malloc((size_t)n_freqs * sizeof(double));
    if (!mag) return ORC_ERR_NOMEM;
    for (int c = 0; c < C; ++c)
        for (long f = 0; f < frames; ++f) {
            long start = f * hop;
            for (int r = 0; r < n_freqs; ++r) {
                double re = 0.0, im = 0.0;
                for (int j = 0; j < L; ++j) {
                    long idx = start + j;
                    double v = 0.0;
                    if (idx >= left && idx - left < T) v = (double)x[(size_t)c * T + (idx - left)];
                    re += v * (double)basis[(size_t)r * L + j];
                    im += v * (double)basis[(size_t)(n_freqs + r) * L + j];
                }
                mag[r] = rnd(sqrt(re * re + im * im), store_f64);
            }
            for (int m = 0; m < n_mels; ++m) {
                double acc = 0.0;
                for (int r = 0; r < n_freqs; ++r)
                    acc += (double)mel_basis[(size_t)m * n_freqs + r] * mag[r];
                out[((size_t)c * n_mels + m) * frames + f] =
                    (float)log(acc > 1e-5 ? acc : 1e-5);
            }
        }
    free(mag);
    return ORC_OK;
}

/* Frames of orc_mel_stft for T samples. */
long orc_mel_frames(int T, int L, int hop) {
    long left = L > hop ? L - hop : 0;
    return (T + left - L) / hop + 1;
}

/* The x ratio Hann-windowed sinc upsampler ([LTX] `hann_sinc_upsample`,
 * rolloff 0.99, window half-width 6 zero crossings): width = ceil(6/0.99),
 * k = 2 width ratio + 1 taps
 *   filt[a] = sinc(ta) cos^2(clamp(ta, -6, 6) pi / 12) 0.99 / ratio,
 *   ta = (a / ratio - width) 0.99,
 * then, on x replicate-padded by `width` samples each side (scaled by ratio),
 * a transposed FIR acc[p ratio + a] += v_p filt[a], trimmed to
 * [2 width ratio, full - (k - ratio)): ratio T samples per row.
 * x [C, T] -> y [C, ratio T]. */
int orc_hann_sinc_upsample(const float *x, int C, int T, int ratio, int store_f64, float *y) {
    if (C <= 0 || T <= 0 || ratio <= 0) return ORC_ERR_ARG;
    const double rolloff = 0.99, lpw = 6.0;
    int width = (int)ceil(lpw / rolloff);
    int k = 2 * width * ratio + 1;
    int pad = width;
    long pad_left = 2L * width * ratio, pad_right = k - ratio;
    double *filt = (double *)malloc((size_t)k * sizeof(double));
    long tp = T + 2L * pad;
    long full = (tp - 1) * ratio + k;
    double *acc = (double *)malloc((size_t)full * sizeof(double));
    if (!filt || !acc) { free(filt); free(acc); return ORC_ERR_NOMEM; }
    for (int a = 0; a < k; ++a) {
        double ta = ((double)a / ratio - width) * rolloff;
        double tc = ta < -lpw ? -lpw : (ta > lpw ? lpw : ta);
        double win = cos(tc * M_PI / lpw / 2.0);
        win *= win;
        double s = ta == 0.0 ? 1.0 : sin(M_PI * ta) / (M_PI * ta);
        filt[a] = (double)(float)(s * win * rolloff / ratio);  /* the page's float taps */
    }
    long t2 = full - pad_right - pad_left;
    for (int c = 0; c < C; ++c) {
        for (long q = 0; q < full; ++q) acc[q] = 0.0;
        for (long p = 0; p < tp; ++p) {
            long src = p - pad;
            src = src < 0 ? 0 : (src > T - 1 ? T - 1 : src);
            double v = (double)x[(size_t)c * T + src] * ratio;
            for (int a = 0; a < k; ++a) acc[p * ratio + a] += v * filt[a];
        }
        for (long i = 0; i < t2; ++i) y[(size_t)c * t2 + i] = (float)rnd(acc[pad_left + i], store_f64);
    }
    free(filt); free(acc);
    return ORC_OK;
}

/* The bandwidth-extension tail ([LTX] `AudioStack::decode_from_mel` after the
 * first generator): low [C, T] at the input rate is zero-padded to a whole
 * number of mel hops, its log-mel (orc_mel_stft, folded) drives the extender
 * (a decoder of geometry g on one row of C n_mels channels, C outputs, no
 * final op -- its output is a residual), the padded low signal is upsampled
 * by `ratio` (orc_hann_sinc_upsample), and
 *   y[c, i] = clamp(residual[c, i] + skip[c, i], -1, 1),  i < ratio T.
 * g's out_channels must be C, in_channels C n_mels and its hop
 * ratio x mel hop. */
int orc_bwe_tail(const int *g, const float *params, const float *low, int C, int T,
                 const float *basis, int n_freqs, int L, int hop, const float *mel_basis,
                 int n_mels, int ratio, const float *up, const float *down, int FK,
                 int store_f64, float *y) {
    if (!geo_ok(g) || C <= 0 || T <= 0 || ratio <= 0) return ORC_ERR_ARG;
    if (g[G_IN] != C * n_mels || g[G_OUT] != C) return ORC_ERR_ARG;
    long ghop = 1;
    for (int i = 0; i < g[G_NUP]; ++i) ghop *= g[G_RATE + i];
    if (ghop != (long)ratio * hop) return ORC_ERR_ARG;
    long Tp = T % hop == 0 ? T : T + hop - T % hop;
    float *padded = (float *)calloc((size_t)C * Tp, sizeof(float));
    long frames = orc_mel_frames((int)Tp, L, hop);
    float *mel = (float *)malloc((size_t)C * n_mels * frames * sizeof(float));
    float *res = (float *)malloc((size_t)C * frames * ghop * sizeof(float));
    float *skip = (float *)malloc((size_t)C * ratio * Tp * sizeof(float));
    int rc = ORC_ERR_NOMEM;
    if (padded && mel && res && skip) {
        for (int c = 0; c < C; ++c)
            memcpy(padded + (size_t)c * Tp, low + (size_t)c * T, (size_t)T * sizeof(float));
        rc = orc_mel_stft(padded, C, (int)Tp, basis, n_freqs, L, hop, mel_basis, n_mels,
                          store_f64, mel);
        if (rc == ORC_OK)
            rc = orc_decode(g, params, mel, 1, (int)frames, up, down, FK, 1e-9, store_f64, res);
        if (rc == ORC_OK) rc = orc_hann_sinc_upsample(padded, C, (int)Tp, ratio, store_f64, skip);
        if (rc == ORC_OK) {
            long n = (long)ratio * T;
            long rt = frames * ghop, st = (long)ratio * Tp;
            for (int c = 0; c < C; ++c)
                for (long i = 0; i < n; ++i) {
                    double v = (double)res[(size_t)c * rt + i] + (double)skip[(size_t)c * st + i];
                    y[(size_t)c * n + i] = (float)(v < -1.0 ? -1.0 : (v > 1.0 ? 1.0 : v));
                }
        }
    }
    free(padded); free(mel); free(res); free(skip);
    return rc;
}
