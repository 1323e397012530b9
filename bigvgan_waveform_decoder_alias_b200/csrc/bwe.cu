// The LTX-2.5 bandwidth-extension tail (docs.rs cortiq-engine 0.6.3
// ltxaudio.rs, `MelStft::forward`, `hann_sinc_upsample` and
// `AudioStack::decode_from_mel`): a 16 kHz signal becomes 48 kHz as
//   clamp(extender(log-mel(low)) + upsample_x3(low), -1, 1),
// where the extender is a BigVGAN v2 generator run by the library's decoder
// on the (channel, mel) fold of the log-mel.
//
// Kernels:
//  - mel_stft_kernel: one CTA per (channel, 8 frames) stages the frames'
//    samples (the causal left pad included) in shared memory; one thread per
//    frequency bin accumulates the window-DFT dot products of all 8 frames
//    (the basis row read once per frame group), the magnitudes meet in shared
//    memory, and the mel bank and log follow in the same CTA.
//  - sinc_upsample_kernel: the transposed FIR as a gather, one output per
//    thread, ceil(k / ratio) taps each.
//  - pad and clamped-sum kernels.
#include <algorithm>
#include <cmath>

#include "common.cuh"

namespace bv {
namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

constexpr int MEL_FB = 8;        // frames per CTA
constexpr int MAX_SINC_TAPS = 256;

long long mel_frames(long long T, int L, int hop) {
  const long long left = L > hop ? L - hop : 0;
  return (T + left - L) / hop + 1;
}

__global__ void mel_stft_kernel(const float *__restrict__ x, int T,
                                const float *__restrict__ basis, int n_freqs, int L, int hop,
                                const float *__restrict__ mel_basis, int n_mels, int frames,
                                float *__restrict__ out) {
  extern __shared__ __align__(16) float sm[];
  const int c = blockIdx.y, f0 = blockIdx.x * MEL_FB;
  const int nf = min(MEL_FB, frames - f0);
  const int left = L > hop ? L - hop : 0;
  const int span = (MEL_FB - 1) * hop + L;
  float *win = sm;                 // [span]: padded-signal samples f0 hop ..
  float *mag = sm + span;          // [n_freqs][MEL_FB]
  const float *xr = x + (size_t)c * T;
  for (int j = threadIdx.x; j < span; j += blockDim.x) {
    const long long idx = (long long)f0 * hop + j - left;  // sample of the unpadded signal
    win[j] = (idx >= 0 && idx < T) ? __ldg(xr + idx) : 0.0f;
  }
  __syncthreads();
  for (int r = threadIdx.x; r < n_freqs; r += blockDim.x) {
    float re[MEL_FB], im[MEL_FB];
#pragma unroll
    for (int f = 0; f < MEL_FB; ++f) re[f] = im[f] = 0.0f;
    const float *br = basis + (size_t)r * L, *bi = basis + (size_t)(n_freqs + r) * L;
    for (int j = 0; j < L; ++j) {
      const float a = __ldg(br + j), b = __ldg(bi + j);
#pragma unroll
      for (int f = 0; f < MEL_FB; ++f) {
        const float v = win[f * hop + j];
        re[f] = fmaf(v, a, re[f]);
        im[f] = fmaf(v, b, im[f]);
      }
    }
#pragma unroll
    for (int f = 0; f < MEL_FB; ++f) mag[r * MEL_FB + f] = sqrtf(re[f] * re[f] + im[f] * im[f]);
  }
  __syncthreads();
  for (int q = threadIdx.x; q < n_mels * nf; q += blockDim.x) {
    const int m = q / nf, f = q - m * nf;
    const float *mr = mel_basis + (size_t)m * n_freqs;
    float acc = 0.0f;
    for (int r = 0; r < n_freqs; ++r) acc = fmaf(__ldg(mr + r), mag[r * MEL_FB + f], acc);
    out[((size_t)c * n_mels + m) * frames + f0 + f] = logf(fmaxf(acc, 1e-5f));
  }
}

struct SincTaps {
  int k, width, ratio;
  float f[MAX_SINC_TAPS];
};

// y[c, i] = sum_p v_p filt[i + 2 width ratio - p ratio], v_p = ratio x[c,
// clamp(p - width, 0, T - 1)], over p in [0, T + 2 width) with the tap index
// in [0, k); rows of y have y_pitch samples, the first n computed.
__global__ void sinc_upsample_kernel(const float *__restrict__ x, int C, int T, SincTaps tp,
                                     float *__restrict__ y, long long n, long long y_pitch) {
  const long long total = (long long)C * n;
  const long long tpl = (long long)T + 2 * tp.width;
  for (long long g = blockIdx.x * (long long)blockDim.x + threadIdx.x; g < total;
       g += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(g / n);
    const long long i = g - (long long)c * n;
    const long long q = i + 2LL * tp.width * tp.ratio;
    long long p0 = q - (tp.k - 1);
    p0 = p0 <= 0 ? 0 : (p0 + tp.ratio - 1) / tp.ratio;
    long long p1 = q / tp.ratio;
    if (p1 > tpl - 1) p1 = tpl - 1;
    const float *xr = x + (size_t)c * T;
    float acc = 0.0f;
    for (long long p = p0; p <= p1; ++p) {
      long long src = p - tp.width;
      src = src < 0 ? 0 : (src > T - 1 ? T - 1 : src);
      acc = fmaf(__ldg(xr + src) * (float)tp.ratio, tp.f[q - p * tp.ratio], acc);
    }
    y[(size_t)c * y_pitch + i] = acc;
  }
}

// y[c, t] = t < T ? x[c, t] : 0 over rows of length Tp.
__global__ void pad_rows_kernel(const float *__restrict__ x, float *__restrict__ y, int C, int T,
                                int Tp) {
  const long long total = (long long)C * Tp;
  for (long long g = blockIdx.x * (long long)blockDim.x + threadIdx.x; g < total;
       g += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(g / Tp), t = (int)(g - (long long)c * Tp);
    y[g] = t < T ? __ldg(x + (size_t)c * T + t) : 0.0f;
  }
}

// y[c, i] = clamp(a[c, i] + b[c, i], -1, 1), i < n (rows: a_pitch, b_pitch, n).
__global__ void add_clamp_kernel(const float *__restrict__ a, long long a_pitch,
                                 const float *__restrict__ b, long long b_pitch,
                                 float *__restrict__ y, int C, long long n) {
  const long long total = (long long)C * n;
  for (long long g = blockIdx.x * (long long)blockDim.x + threadIdx.x; g < total;
       g += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(g / n);
    const long long i = g - (long long)c * n;
    const float v = __ldg(a + (size_t)c * a_pitch + i) + __ldg(b + (size_t)c * b_pitch + i);
    y[g] = fminf(fmaxf(v, -1.0f), 1.0f);
  }
}

unsigned grid_for(long long n) {
  const long long b = (n + 255) / 256;
  return (unsigned)(b < 148 * 16 ? (b > 0 ? b : 1) : 148 * 16);
}

// The page's float taps of the x ratio Hann-windowed sinc (rolloff 0.99,
// 6 zero crossings), computed in double.
bool make_taps(int ratio, SincTaps *t) {
  const double rolloff = 0.99, lpw = 6.0;
  t->ratio = ratio;
  t->width = (int)std::ceil(lpw / rolloff);
  t->k = 2 * t->width * ratio + 1;
  if (t->k > MAX_SINC_TAPS) return false;
  for (int a = 0; a < t->k; ++a) {
    const double ta = ((double)a / ratio - t->width) * rolloff;
    const double tc = std::min(std::max(ta, -lpw), lpw);
    double win = std::cos(tc * M_PI / lpw / 2.0);
    win *= win;
    const double s = ta == 0.0 ? 1.0 : std::sin(M_PI * ta) / (M_PI * ta);
    t->f[a] = (float)(s * win * rolloff / ratio);
  }
  return true;
}

bv_status launch_mel_stft(const float *x, int C, int T, const float *basis, int n_freqs, int L,
                          int hop, const float *mel_basis, int n_mels, float *out,
                          cudaStream_t st) {
  const long long frames = mel_frames(T, L, hop);
  if (frames <= 0) return BV_OK;
  const size_t smem = ((size_t)(MEL_FB - 1) * hop + L + (size_t)n_freqs * MEL_FB) * sizeof(float);
  if (smem > 200 * 1024) return fail(BV_ERR_UNSUPPORTED, "mel_stft: n_fft %d too large", L);
  BV_TRY(ensure_dynamic_smem((const void *)mel_stft_kernel, smem, "mel_stft smem attribute"));
  const int threads = std::min(1024, (n_freqs + 31) / 32 * 32);
  dim3 grid((unsigned)((frames + MEL_FB - 1) / MEL_FB), (unsigned)C);
  if (grid.y > 65535) return fail(BV_ERR_SHAPE, "mel_stft: %d channels", C);
  {
    LaunchTimer tm(st, "mel_stft", 4.0 * C * frames * (double)n_freqs * L,
                   4.0 * ((double)C * T + (double)C * n_mels * frames));
    mel_stft_kernel<<<grid, threads, smem, st>>>(x, T, basis, n_freqs, L, hop, mel_basis, n_mels,
                                                 (int)frames, out);
  }
  count_launch();
  return check_launch("mel_stft_kernel");
}

bv_status launch_sinc_upsample(const float *x, int C, int T, int ratio, float *y, long long n,
                               long long y_pitch, cudaStream_t st) {
  SincTaps taps;
  if (!make_taps(ratio, &taps)) return fail(BV_ERR_UNSUPPORTED, "sinc upsample: ratio %d", ratio);
  const long long total = (long long)C * n;
  if (total <= 0) return BV_OK;
  {
    LaunchTimer tm(st, "sinc_upsample", 2.0 * total * ((taps.k + ratio - 1) / ratio),
                   4.0 * ((double)C * T + (double)total));
    sinc_upsample_kernel<<<grid_for(total), 256, 0, st>>>(x, C, T, taps, y, n, y_pitch);
  }
  count_launch();
  return check_launch("sinc_upsample_kernel");
}

struct TailPlan {
  long long Tp = 0, frames = 0, ghop = 0;
  size_t padded = 0, mel = 0, res = 0, skip = 0, dec = 0, total = 0;
};

bv_status tail_plan(const bv_decoder_config *c, int C, int T, int L, int hop, int n_mels,
                    int ratio, TailPlan *p) {
  if (C < 1 || T < 1 || L < 1 || hop < 1 || n_mels < 1 || ratio < 1 || ratio > 16)
    return fail(BV_ERR_SHAPE, "bwe tail: C=%d T=%d n_fft=%d hop=%d n_mels=%d ratio=%d", C, T, L,
                hop, n_mels, ratio);
  if (c->in_channels != C * n_mels || c->out_channels != C)
    return fail(BV_ERR_SHAPE, "bwe tail: the extender takes %d channels and gives %d; need %d and %d",
                c->in_channels, c->out_channels, C * n_mels, C);
  p->ghop = decoder_hop(c);
  if (p->ghop != (long long)ratio * hop)
    return fail(BV_ERR_SHAPE, "bwe tail: extender hop %lld != ratio %d x mel hop %d", p->ghop,
                ratio, hop);
  p->Tp = (T + hop - 1) / hop * (long long)hop;
  if (p->Tp + (L > hop ? L - hop : 0) < L) return fail(BV_ERR_SHAPE, "bwe tail: signal shorter than a frame");
  p->frames = mel_frames(p->Tp, L, hop);
  p->padded = align_up((size_t)C * p->Tp * sizeof(float));
  p->mel = align_up((size_t)C * n_mels * p->frames * sizeof(float));
  p->res = align_up((size_t)C * p->frames * p->ghop * sizeof(float));
  p->skip = align_up((size_t)C * ratio * T * sizeof(float));
  p->dec = decoder_workspace(c, 1, (int)p->frames);
  if (p->dec == 0) return fail(BV_ERR_SHAPE, "bwe tail: extender workspace");
  p->total = p->padded + p->mel + p->res + p->skip + p->dec;
  return BV_OK;
}

}  // namespace
}  // namespace bv

using namespace bv;

extern "C" {

bv_status bv_mel_stft(const float *x, int C, int T, const float *basis, int n_freqs, int n_fft,
                      int hop, const float *mel_basis, int n_mels, float *out, void *stream) {
  clear_error();
  if (!x || !basis || !mel_basis || !out) return fail(BV_ERR_ARG, "bv_mel_stft: null pointer");
  if (C < 1 || T < 1 || n_freqs < 1 || n_fft < 1 || hop < 1 || n_mels < 1 ||
      mel_frames(T, n_fft, hop) < 1)
    return fail(BV_ERR_SHAPE, "bv_mel_stft: C=%d T=%d n_freqs=%d n_fft=%d hop=%d n_mels=%d", C,
                T, n_freqs, n_fft, hop, n_mels);
  BV_TRY(require_device());
  return launch_mel_stft(x, C, T, basis, n_freqs, n_fft, hop, mel_basis, n_mels, out,
                         as_stream(stream));
}

int64_t bv_mel_frames(int T, int n_fft, int hop) {
  if (T < 1 || n_fft < 1 || hop < 1) return -1;
  return mel_frames(T, n_fft, hop);
}

bv_status bv_sinc_upsample(const float *x, int C, int T, int ratio, float *y, void *stream) {
  clear_error();
  if (!x || !y) return fail(BV_ERR_ARG, "bv_sinc_upsample: null pointer");
  if (C < 1 || T < 1 || ratio < 1 || ratio > 16)
    return fail(BV_ERR_SHAPE, "bv_sinc_upsample: C=%d T=%d ratio=%d", C, T, ratio);
  if (overlaps(x, (size_t)C * T, y, (size_t)C * ratio * T))
    return fail(BV_ERR_ARG, "bv_sinc_upsample: x and y overlap");
  BV_TRY(require_device());
  return launch_sinc_upsample(x, C, T, ratio, y, (long long)ratio * T, (long long)ratio * T,
                              as_stream(stream));
}

size_t bv_bwe_tail_workspace_size(const bv_decoder_config *cfg, int C, int T, int n_fft,
                                  int hop, int n_mels, int ratio) {
  clear_error();
  if (!cfg) return 0;
  TailPlan p;
  if (tail_plan(cfg, C, T, n_fft, hop, n_mels, ratio, &p) != BV_OK) return 0;
  return p.total;
}

bv_status bv_bwe_tail(const bv_decoder_config *cfg, const bv_decoder_weights *w, const float *low,
                      int C, int T, const float *stft_basis, int n_fft, int hop,
                      const float *mel_basis, int n_mels, int ratio, float *y, void *workspace,
                      size_t ws_bytes, void *stream) {
  clear_error();
  if (!low || !y || !stft_basis || !mel_basis) return fail(BV_ERR_ARG, "bv_bwe_tail: null pointer");
  BV_TRY(decoder_check(cfg, w));
  if (cfg->tile_frames != 0 || cfg->latent_channels != 0)
    return fail(BV_ERR_ARG, "bv_bwe_tail: the extender config is untiled and without front end");
  TailPlan p;
  BV_TRY(tail_plan(cfg, C, T, n_fft, hop, n_mels, ratio, &p));
  if (!workspace || ws_bytes < p.total)
    return fail(BV_ERR_WORKSPACE, "bv_bwe_tail: workspace %zu bytes, need %zu", ws_bytes, p.total);
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return fail(BV_ERR_ARG, "bv_bwe_tail: workspace not 256-byte aligned");
  const size_t nl = (size_t)C * T, ny = (size_t)C * ratio * T;
  const float *wsf = static_cast<const float *>(workspace);
  if (overlaps(low, nl, y, ny) || overlaps(low, nl, wsf, p.total / 4) ||
      overlaps(y, ny, wsf, p.total / 4))
    return fail(BV_ERR_ARG, "bv_bwe_tail: low, y and workspace must be disjoint");
  BV_TRY(require_device());
  cudaStream_t st = as_stream(stream);
  char *ws = static_cast<char *>(workspace);
  float *padded = reinterpret_cast<float *>(ws);
  float *mel = reinterpret_cast<float *>(ws + p.padded);
  float *res = reinterpret_cast<float *>(ws + p.padded + p.mel);
  float *skip = reinterpret_cast<float *>(ws + p.padded + p.mel + p.res);
  char *dec_ws = ws + p.padded + p.mel + p.res + p.skip;
  const int n_freqs = n_fft / 2 + 1;
  // zero-pad the low signal to whole mel hops
  {
    LaunchTimer tm(st, "bwe_glue", 0.0, 4.0 * ((double)nl + (double)C * p.Tp));
    pad_rows_kernel<<<grid_for((long long)C * p.Tp), 256, 0, st>>>(low, padded, C, T, (int)p.Tp);
  }
  count_launch();
  BV_TRY(check_launch("pad_rows_kernel"));
  BV_TRY(launch_mel_stft(padded, C, (int)p.Tp, stft_basis, n_freqs, n_fft, hop, mel_basis, n_mels,
                         mel, st));
  // the extender on the folded mel: one row of C n_mels channels, C outputs
  BV_TRY(decoder_run(cfg, w, mel, 1, (int)p.frames, res, dec_ws, st));
  // the skip path and the clamped sum over the first ratio T samples
  const long long n = (long long)ratio * T;
  BV_TRY(launch_sinc_upsample(padded, C, (int)p.Tp, ratio, skip, n, n, st));
  {
    LaunchTimer tm(st, "bwe_glue", 0.0, 12.0 * (double)C * n);
    add_clamp_kernel<<<grid_for((long long)C * n), 256, 0, st>>>(res, p.frames * p.ghop, skip, n,
                                                                  y, C, n);
  }
  count_launch();
  return check_launch("add_clamp_kernel");
}

}  // extern "C"
