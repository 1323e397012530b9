// The C ABI of libbv: argument checks, the filter design, and the host-side
// orchestration of the AMP block and the decoder.  Every step of the
// computation runs in the CUDA kernels of this library.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "bv.h"
#include "common.cuh"
#include "tiles.cuh"

#define BV_VERSION "bv 0.1.0 (sm_100a)"

namespace bv {

namespace {
thread_local char g_err[512] = "";
uint64_t g_launches = 0;
}  // namespace

__device__ int g_device_status = 0;

namespace {
constexpr long long kDefaultWaitLimit = 1ll << 26;
std::atomic<long long> g_wait_limit{kDefaultWaitLimit};
}  // namespace

long long wait_limit() { return g_wait_limit.load(std::memory_order_relaxed); }

int *device_status_ptr() {
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
  return static_cast<int *>(p);
}

bv_status fail(bv_status st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

bv_status check_launch(const char *what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(BV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return BV_OK;
}

void count_launch(uint64_t n) { __atomic_fetch_add(&g_launches, n, __ATOMIC_RELAXED); }

namespace {
struct SmemLimit {
  int dev;
  const void *func;
  size_t bytes;
};
std::mutex g_smem_mu;
std::vector<SmemLimit> g_smem_limits;
}  // namespace

bv_status ensure_dynamic_smem(const void *func, size_t bytes, const char *what) {
  if (bytes <= 48 * 1024) return BV_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return check_launch(what);
  std::lock_guard<std::mutex> lk(g_smem_mu);
  for (SmemLimit &l : g_smem_limits)
    if (l.dev == dev && l.func == func) {
      if (l.bytes >= bytes) return BV_OK;
      if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
          cudaSuccess)
        return check_launch(what);
      l.bytes = bytes;
      return BV_OK;
    }
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
      cudaSuccess)
    return check_launch(what);
  g_smem_limits.push_back({dev, func, bytes});
  return BV_OK;
}

// ------------------------------------------------------------ launch timing

namespace {
struct TimerRec {
  std::string cls;
  cudaEvent_t start = nullptr, stop = nullptr;
  double flops = 0, bytes = 0;
  bool used = false;
};
std::atomic<bool> g_timing_on{false};
std::mutex g_timer_mu;
std::vector<TimerRec> g_timers;
size_t g_timer_next = 0;  // records [0, next) are live
}  // namespace

LaunchTimer::LaunchTimer(cudaStream_t st, const char *cls, double flops, double bytes) : st_(st) {
  if (!g_timing_on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_timer_mu);
  if (g_timer_next == g_timers.size()) {
    TimerRec r;
    if (cudaEventCreate(&r.start) != cudaSuccess || cudaEventCreate(&r.stop) != cudaSuccess) {
      cudaGetLastError();
      return;
    }
    g_timers.push_back(r);
  }
  TimerRec &r = g_timers[g_timer_next];
  r.cls = cls;
  r.flops = flops;
  r.bytes = bytes;
  r.used = true;
  slot_ = (int)g_timer_next++;
  cudaEventRecord(r.start, st_);
}

LaunchTimer::~LaunchTimer() {
  if (slot_ < 0) return;
  std::lock_guard<std::mutex> lk(g_timer_mu);
  cudaEventRecord(g_timers[slot_].stop, st_);
}

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

// The current device must be an sm_100 part; checked once per device.
bv_status check_device() {
  static int ok_mask = 0;  // bit per device id < 32 that passed
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(BV_ERR_CUDA, "no CUDA device: %s", cudaGetErrorString(e));
  if (dev < 32 && (ok_mask >> dev) & 1) return BV_OK;
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10)
    return fail(BV_ERR_CUDA, "device %d is sm_%d%d; this library is built for sm_100a", dev,
                major, minor);
  if (dev < 32) ok_mask |= 1 << dev;
  return BV_OK;
}

// ------------------------------------------------------------- filter design

// Modified Bessel I0 by its power series; terms (x/2)^{2k}/(k!)^2 accumulate
// until they fall below 1e-18 of the sum (at most 39 of them).
double bessel_i0(double x) {
  double s = 1.0, term = 1.0;
  const double h = 0.5 * x;
  for (int k = 1; k <= 39; ++k) {
    term *= (h / k) * (h / k);
    s += term;
    if (term < 1e-18 * s) break;
  }
  return s;
}

double sinc_pi(double v) { return v == 0.0 ? 1.0 : std::sin(M_PI * v) / (M_PI * v); }

}  // namespace

void clear_error() { g_err[0] = 0; }
bv_status require_device() { return check_device(); }

}  // namespace bv

using namespace bv;

extern "C" {

const char *bv_last_error(void) { return g_err; }

const char *bv_version(void) { return BV_VERSION; }

uint64_t bv_launch_count(void) { return __atomic_load_n(&g_launches, __ATOMIC_RELAXED); }

void bv_timing_enable(int on) { g_timing_on.store(on != 0); }

void bv_timing_reset(void) {
  std::lock_guard<std::mutex> lk(g_timer_mu);
  g_timer_next = 0;
}

int bv_timing_read(bv_kernel_stats *out, int max) {
  std::lock_guard<std::mutex> lk(g_timer_mu);
  std::map<std::string, bv_kernel_stats> acc;
  for (size_t i = 0; i < g_timer_next; ++i) {
    TimerRec &r = g_timers[i];
    if (cudaEventSynchronize(r.stop) != cudaSuccess) return -1;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) return -1;
    bv_kernel_stats &k = acc[r.cls];
    if (k.launches == 0) {
      std::memset(&k, 0, sizeof(k));
      snprintf(k.name, sizeof(k.name), "%s", r.cls.c_str());
    }
    k.launches += 1;
    k.ms += ms;
    k.flops += r.flops;
    k.bytes += r.bytes;
  }
  int n = 0;
  for (auto &kv : acc) {
    if (n < max && out) out[n] = kv.second;
    ++n;
  }
  return n;
}

long long bv_debug_set_wait_limit(long long polls) {
  return g_wait_limit.exchange(polls < 0 ? kDefaultWaitLimit : polls);
}

bv_status bv_sync_status(void *stream) {
  g_err[0] = 0;
  BV_TRY(check_device());
  int h = 0;
  cudaStream_t st = as_stream(stream);
  cudaError_t e = cudaMemcpyFromSymbolAsync(&h, g_device_status, sizeof(int), 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(BV_ERR_CUDA, "bv_sync_status: %s", cudaGetErrorString(e));
  if (h != 0) {
    const int zero = 0;
    cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
    cudaStreamSynchronize(st);
    if (h == kStatusF16Range)
      return fail(BV_ERR_RANGE, "an activation reached fp16's range on the fp16 conv path");
    return fail(BV_ERR_TIMEOUT, "a bounded device wait gave up (code %d)", h);
  }
  return BV_OK;
}

bv_status bv_filter_design(double cutoff, double half_width, int taps, float *out_host) {
  g_err[0] = 0;
  if (!out_host) return fail(BV_ERR_ARG, "bv_filter_design: null output");
  if (taps < 1 || taps > 64) return fail(BV_ERR_ARG, "bv_filter_design: taps %d", taps);
  if (!(cutoff > 0.0 && cutoff <= 0.5) || !(half_width > 0.0))
    return fail(BV_ERR_ARG, "bv_filter_design: cutoff %g half_width %g", cutoff, half_width);
  // Kaiser's attenuation estimate and beta for a transition of 4 half_width
  const int half = taps / 2;
  const double atten = 2.285 * (half - 1) * M_PI * (4.0 * half_width) + 7.95;
  double beta = 0.0;
  if (atten > 50.0) beta = 0.1102 * (atten - 8.7);
  else if (atten >= 21.0) beta = 0.5842 * std::pow(atten - 21.0, 0.4) + 0.07886 * (atten - 21.0);
  const double i0b = bessel_i0(beta);
  const double centre = (taps % 2 == 0) ? half - 0.5 : (double)half;
  std::vector<double> f(taps);
  double total = 0.0;
  for (int i = 0; i < taps; ++i) {
    const double r = taps > 1 ? 2.0 * i / (taps - 1) - 1.0 : 0.0;
    const double win = bessel_i0(beta * std::sqrt(std::fmax(0.0, 1.0 - r * r))) / i0b;
    f[i] = 2.0 * cutoff * win * sinc_pi(2.0 * cutoff * (i - centre));
    total += f[i];
  }
  for (int i = 0; i < taps; ++i) out_host[i] = (float)(f[i] / total);
  return BV_OK;
}

bv_status bv_activation1d(const float *x, float *y, int B, int C, int T, const float *log_alpha,
                          const float *log_beta, const float *up_filter,
                          const float *down_filter, float eps, void *stream) {
  g_err[0] = 0;
  if (!x || !y || !log_alpha || !log_beta || !up_filter || !down_filter)
    return fail(BV_ERR_ARG, "bv_activation1d: null pointer");
  if (B < 1 || C < 1 || T < 1) return fail(BV_ERR_SHAPE, "bv_activation1d: B=%d C=%d T=%d", B, C, T);
  const size_t n = (size_t)B * C * T;
  if (n >= (1ull << 40)) return fail(BV_ERR_SHAPE, "bv_activation1d: tensor too large");
  if (!aligned4(x) || !aligned4(y)) return fail(BV_ERR_ARG, "bv_activation1d: misaligned pointer");
  if (overlaps(x, n, y, n)) return fail(BV_ERR_ARG, "bv_activation1d: x and y overlap");
  BV_TRY(check_device());
  return launch_activation(x, y, B, C, T, log_alpha, log_beta, up_filter, down_filter, eps,
                           as_stream(stream));
}

bv_status bv_sin_squared(const float *z, float *out, int64_t n, void *stream) {
  g_err[0] = 0;
  if (!z || !out) return fail(BV_ERR_ARG, "bv_sin_squared: null pointer");
  if (n < 0) return fail(BV_ERR_SHAPE, "bv_sin_squared: n=%lld", (long long)n);
  if (z != out && overlaps(z, (size_t)n, out, (size_t)n))
    return fail(BV_ERR_ARG, "bv_sin_squared: z and out partially overlap");
  BV_TRY(check_device());
  return launch_sin_squared(z, out, n, as_stream(stream));
}

bv_status bv_conv1d(const float *x, int B, int Cin, int T, const float *w, const float *bias,
                    int Cout, int K, int dilation, int pad, const bv_epilogue *ep, float *y,
                    void *stream) {
  g_err[0] = 0;
  if (!x || !w || !y) return fail(BV_ERR_ARG, "bv_conv1d: null pointer");
  if (B < 1 || Cin < 1 || T < 1 || Cout < 1 || K < 1 || K > 32 || dilation < 1 || pad < 0)
    return fail(BV_ERR_SHAPE, "bv_conv1d: B=%d Cin=%d T=%d Cout=%d K=%d d=%d pad=%d", B, Cin, T,
                Cout, K, dilation, pad);
  const long long Tout = (long long)T + 2LL * pad - (long long)dilation * (K - 1);
  if (Tout < 1 || Tout > 0x7fffffffLL) return fail(BV_ERR_SHAPE, "bv_conv1d: output length %lld", Tout);
  const size_t nin = (size_t)B * Cin * T, nout = (size_t)B * Cout * Tout;
  if (overlaps(x, nin, y, nout)) return fail(BV_ERR_ARG, "bv_conv1d: x and y overlap");
  Epi e{nullptr, 1.0f, 0, 0};
  if (ep) {
    e.residual = ep->residual;
    e.scale = ep->scale;
    e.accumulate = ep->accumulate ? 1 : 0;
    e.final_act = ep->final_act;
    if (e.final_act < 0 || e.final_act > 2) return fail(BV_ERR_ARG, "bv_conv1d: final_act %d", e.final_act);
    if (e.residual && e.residual != y && overlaps(e.residual, nout, y, nout))
      return fail(BV_ERR_ARG, "bv_conv1d: residual partially overlaps y");
  }
  BV_TRY(check_device());
  return launch_conv1d(x, B, Cin, T, w, bias, Cout, K, dilation, pad, e, y, (int)Tout, (int)Tout,
                       as_stream(stream));
}

bv_status bv_conv_transpose1d(const float *x, int B, int Cin, int T, const float *w,
                              const float *bias, int Cout, int K, int stride, int pad, float *y,
                              void *stream) {
  g_err[0] = 0;
  if (!x || !w || !y) return fail(BV_ERR_ARG, "bv_conv_transpose1d: null pointer");
  if (B < 1 || Cin < 1 || T < 1 || Cout < 1 || K < 1 || K > 64 || stride < 1 || stride > 16 ||
      pad < 0)
    return fail(BV_ERR_SHAPE, "bv_conv_transpose1d: B=%d Cin=%d T=%d Cout=%d K=%d s=%d pad=%d",
                B, Cin, T, Cout, K, stride, pad);
  const long long Tout = (long long)(T - 1) * stride + K - 2LL * pad;
  if (Tout < 1 || Tout > 0x7fffffffLL)
    return fail(BV_ERR_SHAPE, "bv_conv_transpose1d: output length %lld", Tout);
  if (overlaps(x, (size_t)B * Cin * T, y, (size_t)B * Cout * Tout))
    return fail(BV_ERR_ARG, "bv_conv_transpose1d: x and y overlap");
  BV_TRY(check_device());
  return launch_conv_transpose1d(x, B, Cin, T, w, bias, Cout, K, stride, pad, y,
                                 as_stream(stream));
}

}  // extern "C"

// ------------------------------------------------------------- AMP block

namespace bv {
namespace {

bv_status check_amp_params(const bv_amp_params *p, int C) {
  (void)C;
  if (!p) return fail(BV_ERR_ARG, "amp block: null params");
  if (p->kernel_size < 1 || p->kernel_size % 2 == 0 || p->kernel_size > 32)
    return fail(BV_ERR_SHAPE, "amp block: kernel_size %d (odd, <= 31)", p->kernel_size);
  if (p->n_dilations < 1 || p->n_dilations > BV_MAX_DIL)
    return fail(BV_ERR_SHAPE, "amp block: n_dilations %d", p->n_dilations);
  if (!p->up_filter || !p->down_filter) return fail(BV_ERR_ARG, "amp block: null filter");
  for (int u = 0; u < p->n_dilations; ++u) {
    if (p->dilation[u] < 1) return fail(BV_ERR_SHAPE, "amp block: dilation %d", p->dilation[u]);
    if (!p->conv1_w[u] || !p->conv2_w[u] || !p->act_log_alpha[2 * u] ||
        !p->act_log_beta[2 * u] || !p->act_log_alpha[2 * u + 1] || !p->act_log_beta[2 * u + 1])
      return fail(BV_ERR_ARG, "amp block: null weight in unit %d", u);
  }
  return BV_OK;
}

// xhi / xlo: two [B, T, C] planes for the time-major tensor-core convs
// (nullptr: every conv reads h1 in [B, C, T]).
struct AmpScratch {
  float *cur, *h1, *h2;
  float *xhi = nullptr, *xlo = nullptr;
};

// Pre-split tensor-core weights of one AMP block's convs (nullptr: the conv
// splits its own weights); tm marks tap-major weights for the time-major conv.
struct AmpSplit {
  const float *conv1[BV_MAX_DIL], *conv2[BV_MAX_DIL];
  bool tm1[BV_MAX_DIL], tm2[BV_MAX_DIL];
  bool f16;  // the time-major splits are fp16 (tm_f16_ok and the config allow)
};

// One activation followed by one conv (Cin = C, output length Tout): through
// the time-major planes xhi / xlo when they and tap-major split weights are
// given, else through h1 ([B, C, T]) and the conv kernels that read it.
bv_status act_conv_core(const float *in, int B, int C, int T, const float *la, const float *lb,
                        const float *fu, const float *fd, float eps, const float *w,
                        const float *bias, int Cout, int K, int dil, int pad, const float *w_split,
                        bool tm, const Epi &ep, float *out, int Tout, float *h1, float *xhi,
                        float *xlo, cudaStream_t st, bool f16) {
  if (tm && w_split && xhi) {
    // the activation writes the conv's time-major operand planes itself, in
    // fp16 when the weights were split in fp16 (f16: tm_f16_ok(C))
    if (activation_tm_supported(C)) {
      BV_TRY(launch_activation_tm(in, xhi, xlo, B, C, T, la, lb, fu, fd, eps, st, f16));
    } else {
      BV_TRY(launch_activation(in, h1, B, C, T, la, lb, fu, fd, eps, st));
      BV_TRY(launch_transpose_split(h1, xhi, xlo, B, C, T, st));
    }
    return launch_conv1d_tm(xhi, xlo, B, C, T, w_split, bias, Cout, K, dil, pad, ep, out, Tout,
                            Tout, st, f16);
  }
  // (tap-major split weights, tf32 or fp16, are for the time-major kernel
  // only: without its planes the conv takes the raw weights)
  BV_TRY(launch_activation(in, h1, B, C, T, la, lb, fu, fd, eps, st));
  return launch_conv1d(h1, B, C, T, w, bias, Cout, K, dil, pad, ep, out, Tout, Tout, st,
                       tm ? nullptr : w_split);
}

// act -> conv inside an AMP block (length-preserving pad).
bv_status act_conv(const float *in, int B, int C, int T, const float *la, const float *lb,
                   const bv_amp_params &p, const float *w, const float *bias, const float *w_split,
                   bool tm, int dil, const Epi &ep, float *out, const AmpScratch &s,
                   cudaStream_t st, bool f16) {
  const int K = p.kernel_size, pad = (K * dil - dil) / 2;
  return act_conv_core(in, B, C, T, la, lb, p.up_filter, p.down_filter, 1e-9f, w, bias, C, K, dil,
                       pad, w_split, tm, ep, out, T, s.h1, s.xhi, s.xlo, st, f16);
}

// y = (accumulate ? y : 0) + scale * AMP(x); x, y and the scratch are disjoint.
bv_status run_amp_block(const float *x, int B, int C, int T, const bv_amp_params &p, float *y,
                        float scale, int accumulate, const AmpScratch &s, cudaStream_t st,
                        const AmpSplit *sp = nullptr) {
  const int n = p.n_dilations;
  for (int u = 0; u < n; ++u) {
    const float *src = (u == 0) ? x : s.cur;
    const Epi plain{nullptr, 1.0f, 0, 0};
    BV_TRY(act_conv(src, B, C, T, p.act_log_alpha[2 * u], p.act_log_beta[2 * u], p, p.conv1_w[u],
                    p.conv1_b[u], sp ? sp->conv1[u] : nullptr, sp && sp->tm1[u], p.dilation[u],
                    plain, s.h2, s, st, sp && sp->f16));
    // last unit: y (+)= scale (src + conv2(...)); otherwise cur = src + conv2(...),
    // where src may be cur itself
    const bool last = (u == n - 1);
    const Epi res = last ? Epi{src, scale, accumulate, 0} : Epi{src, 1.0f, 0, 0};
    BV_TRY(act_conv(s.h2, B, C, T, p.act_log_alpha[2 * u + 1], p.act_log_beta[2 * u + 1], p,
                    p.conv2_w[u], p.conv2_b[u], sp ? sp->conv2[u] : nullptr, sp && sp->tm2[u], 1,
                    res, last ? y : s.cur, s, st, sp && sp->f16));
  }
  return BV_OK;
}

// Split-weight bytes of an AMP block's time-major tensor-core convs (0 when
// none qualifies): tf32 hi / lo of each tap-major [C, K, Cp] matrix.
size_t amp_split_bytes(int C, const bv_amp_params &p) {
  const int K = p.kernel_size;
  size_t s = 0;
  for (int u = 0; u < p.n_dilations; ++u) {
    if (conv1d_tm_supported(C, C, K, p.dilation[u]))
      s += align_up(2 * (size_t)tm_cin_pad(C) * C * K * sizeof(float));
    if (conv1d_tm_supported(C, C, K, 1))
      s += align_up(2 * (size_t)tm_cin_pad(C) * C * K * sizeof(float));
  }
  return s;
}

// Write the split weights of the block's time-major convs into ws (laid out
// as amp_split_bytes counts them) and point `out` at them.
bv_status split_amp_weights(int C, const bv_amp_params &p, char *ws, AmpSplit *out,
                            cudaStream_t st) {
  const int K = p.kernel_size;
  SplitTable tab;
  tab.n = 0;
  size_t off = 0;
  auto add = [&](const float *src, const float **slot, bool *tm) {
    float *dst = reinterpret_cast<float *>(ws + off);
    off += align_up(2 * (size_t)tm_cin_pad(C) * C * K * sizeof(float));
    *slot = dst;
    *tm = true;
    tab.src[tab.n] = src;
    tab.dst[tab.n] = dst;
    tab.count[tab.n] = (long long)C * C * K;
    tab.cin[tab.n] = C;
    tab.k[tab.n] = K;
    tab.f16[tab.n] = out->f16;
    ++tab.n;
  };
  out->f16 = tm_f16_ok(C);
  for (int u = 0; u < p.n_dilations; ++u) {
    if (conv1d_tm_supported(C, C, K, p.dilation[u])) add(p.conv1_w[u], &out->conv1[u], &out->tm1[u]);
    if (conv1d_tm_supported(C, C, K, 1)) add(p.conv2_w[u], &out->conv2[u], &out->tm2[u]);
  }
  return launch_split_weights(tab, st);
}

}  // namespace
}  // namespace bv

extern "C" {

size_t bv_amp_block_workspace_size(int B, int C, int T) {
  if (B < 1 || C < 1 || T < 1) return 0;
  return 3 * align_up((size_t)B * C * T * sizeof(float));
}

size_t bv_amp_block_workspace_size_tc(int B, int C, int T, const bv_amp_params *p) {
  g_err[0] = 0;
  if (B < 1 || C < 1 || T < 1 || check_amp_params(p, C) != BV_OK) return 0;
  const size_t base = bv_amp_block_workspace_size(B, C, T);
  const size_t split = bv::amp_split_bytes(C, *p);
  if (split == 0) return base;
  return base + 2 * bv::align_up((size_t)B * C * T * sizeof(float)) + split;
}

bv_status bv_amp_block(const float *x, int B, int C, int T, const bv_amp_params *p, float *y,
                       float scale, int accumulate, void *workspace, size_t ws_bytes,
                       void *stream) {
  g_err[0] = 0;
  if (!x || !y) return fail(BV_ERR_ARG, "bv_amp_block: null x or y");
  if (B < 1 || C < 1 || T < 1) return fail(BV_ERR_SHAPE, "bv_amp_block: B=%d C=%d T=%d", B, C, T);
  BV_TRY(check_amp_params(p, C));
  const size_t n = (size_t)B * C * T;
  const size_t need = bv_amp_block_workspace_size(B, C, T);
  if (!workspace || ws_bytes < need)
    return fail(BV_ERR_WORKSPACE, "bv_amp_block: workspace %zu bytes, need %zu", ws_bytes, need);
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return fail(BV_ERR_ARG, "bv_amp_block: workspace not 256-byte aligned");
  BV_TRY(check_device());
  const size_t sz = align_up(n * sizeof(float));
  const size_t split = amp_split_bytes(C, *p);
  const bool tc = split > 0 && ws_bytes >= need + 2 * sz + split;  // time-major path fits
  const size_t used = tc ? need + 2 * sz + split : need;
  const float *wsf = static_cast<const float *>(workspace);
  if (overlaps(x, n, y, n) || overlaps(x, n, wsf, used / 4) || overlaps(y, n, wsf, used / 4))
    return fail(BV_ERR_ARG, "bv_amp_block: x, y and workspace must be disjoint");
  char *w8 = static_cast<char *>(workspace);
  AmpScratch s{reinterpret_cast<float *>(w8), reinterpret_cast<float *>(w8 + sz),
               reinterpret_cast<float *>(w8 + 2 * sz)};
  cudaStream_t st = as_stream(stream);
  if (tc) {
    // time-major tensor-core path: operand planes, then the split weights
    s.xhi = reinterpret_cast<float *>(w8 + 3 * sz);
    s.xlo = reinterpret_cast<float *>(w8 + 4 * sz);
    AmpSplit sp{};
    BV_TRY(split_amp_weights(C, *p, w8 + 5 * sz, &sp, st));
    return run_amp_block(x, B, C, T, *p, y, scale, accumulate, s, st, &sp);
  }
  return run_amp_block(x, B, C, T, *p, y, scale, accumulate, s, st);
}

}  // extern "C"

// ------------------------------------ one layer on the decoder's own kernels

namespace bv {
namespace {

// Workspace of bv_act_conv1d: the activation's [B, C, T] output; when the
// conv qualifies for the time-major tensor-core path, also two [B, T, C]
// operand planes and the weights split tap-major into tf32 hi / lo.
struct ActConvPlan {
  bool tm = false;
  size_t h1 = 0, plane = 0, split = 0, total = 0;
};

ActConvPlan act_conv_plan(int B, int C, int T, int Cout, int K, int dil) {
  ActConvPlan p;
  const size_t n = (size_t)B * C * T;
  p.tm = conv1d_tm_supported(C, Cout, K, dil);
  p.h1 = align_up(n * sizeof(float));
  if (p.tm) {
    p.plane = align_up(n * sizeof(float));
    p.split = align_up(2 * (size_t)tm_cin_pad(C) * Cout * K * sizeof(float));
  }
  p.total = p.h1 + 2 * p.plane + p.split;
  return p;
}

// Workspace of bv_conv_transpose1d_ws: the time-major planes and the phase
// weights of the time-major kernel, or the phase weights of the [B, C, T]
// tensor-core kernel, or nothing (FP32 kernel).
struct ConvTPlan {
  int path = 0;  // 2 time-major, 1 [B, C, T] tensor cores, 0 FP32
  size_t plane = 0, wp = 0, total = 0;
};

ConvTPlan convt_plan(int B, int Cin, int T, int Cout, int K, int S) {
  ConvTPlan p;
  if (conv_transpose1d_tm_supported(Cin, Cout, K, S)) {
    p.path = 2;
    p.plane = align_up((size_t)B * Cin * T * sizeof(float));
    p.wp = align_up(conv_transpose1d_tm_workspace(Cin, Cout, K, S));
  } else if (conv_transpose1d_tc_supported(Cin, Cout, K, S)) {
    p.path = 1;
    p.wp = align_up(conv_transpose1d_tc_workspace(Cin, Cout, K, S));
  }
  p.total = 2 * p.plane + p.wp;
  return p;
}

}  // namespace
}  // namespace bv

extern "C" {

size_t bv_act_conv1d_workspace_size(int B, int C, int T, int Cout, int K, int dilation) {
  if (B < 1 || C < 1 || T < 1 || Cout < 1 || K < 1 || K > 32 || dilation < 1) return 0;
  return act_conv_plan(B, C, T, Cout, K, dilation).total;
}

bv_status bv_act_conv1d(const float *x, int B, int C, int T, const float *log_alpha,
                        const float *log_beta, const float *up_filter, const float *down_filter,
                        float eps, const float *w, const float *bias, int Cout, int K,
                        int dilation, int pad, const bv_epilogue *ep, float *y, void *workspace,
                        size_t ws_bytes, void *stream) {
  g_err[0] = 0;
  if (!x || !y || !w || !log_alpha || !log_beta || !up_filter || !down_filter)
    return fail(BV_ERR_ARG, "bv_act_conv1d: null pointer");
  if (B < 1 || C < 1 || T < 1 || Cout < 1 || K < 1 || K > 32 || dilation < 1 || pad < 0)
    return fail(BV_ERR_SHAPE, "bv_act_conv1d: B=%d C=%d T=%d Cout=%d K=%d d=%d pad=%d", B, C, T,
                Cout, K, dilation, pad);
  const long long Tout = (long long)T + 2LL * pad - (long long)dilation * (K - 1);
  if (Tout < 1 || Tout > 0x7fffffffLL)
    return fail(BV_ERR_SHAPE, "bv_act_conv1d: output length %lld", Tout);
  const size_t nin = (size_t)B * C * T, nout = (size_t)B * Cout * Tout;
  if (nin >= (1ull << 40)) return fail(BV_ERR_SHAPE, "bv_act_conv1d: tensor too large");
  Epi e{nullptr, 1.0f, 0, 0};
  if (ep) {
    e = Epi{ep->residual, ep->scale, ep->accumulate ? 1 : 0, ep->final_act};
    if (e.final_act < 0 || e.final_act > 2)
      return fail(BV_ERR_ARG, "bv_act_conv1d: final_act %d", e.final_act);
  }
  const ActConvPlan plan = act_conv_plan(B, C, T, Cout, K, dilation);
  if (!workspace || ws_bytes < plan.total)
    return fail(BV_ERR_WORKSPACE, "bv_act_conv1d: workspace %zu bytes, need %zu", ws_bytes,
                plan.total);
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return fail(BV_ERR_ARG, "bv_act_conv1d: workspace not 256-byte aligned");
  if (!aligned4(x) || !aligned4(y)) return fail(BV_ERR_ARG, "bv_act_conv1d: misaligned pointer");
  const float *wsf = static_cast<const float *>(workspace);
  const size_t nws = plan.total / sizeof(float);
  if (overlaps(x, nin, y, nout) || overlaps(x, nin, wsf, nws) || overlaps(y, nout, wsf, nws))
    return fail(BV_ERR_ARG, "bv_act_conv1d: x, y and workspace must be disjoint");
  if (e.residual && ((e.residual != y && overlaps(e.residual, nout, y, nout)) ||
                     overlaps(e.residual, nout, wsf, nws)))
    return fail(BV_ERR_ARG, "bv_act_conv1d: residual partially overlaps y or the workspace");
  BV_TRY(check_device());
  cudaStream_t st = as_stream(stream);
  char *w8 = static_cast<char *>(workspace);
  float *h1 = reinterpret_cast<float *>(w8);
  float *xhi = nullptr, *xlo = nullptr, *split = nullptr;
  if (plan.tm) {
    xhi = reinterpret_cast<float *>(w8 + plan.h1);
    xlo = reinterpret_cast<float *>(w8 + plan.h1 + plan.plane);
    split = reinterpret_cast<float *>(w8 + plan.h1 + 2 * plan.plane);
    SplitTable tab;
    tab.n = 1;
    tab.src[0] = w;
    tab.dst[0] = split;
    tab.count[0] = (long long)Cout * C * K;
    tab.cin[0] = C;
    tab.k[0] = K;
    tab.f16[0] = tm_f16_ok(C);
    BV_TRY(launch_split_weights(tab, st));
  }
  return act_conv_core(x, B, C, T, log_alpha, log_beta, up_filter, down_filter, eps, w, bias,
                       Cout, K, dilation, pad, split, plan.tm, e, y, (int)Tout, h1, xhi, xlo, st,
                       plan.tm && tm_f16_ok(C));
}

size_t bv_conv_transpose1d_workspace_size(int B, int Cin, int T, int Cout, int K, int stride) {
  if (B < 1 || Cin < 1 || T < 1 || Cout < 1 || K < 1 || K > 64 || stride < 1 || stride > 16)
    return 0;
  return convt_plan(B, Cin, T, Cout, K, stride).total;
}

bv_status bv_conv_transpose1d_ws(const float *x, int B, int Cin, int T, const float *w,
                                 const float *bias, int Cout, int K, int stride, int pad,
                                 float *y, void *workspace, size_t ws_bytes, void *stream) {
  g_err[0] = 0;
  if (!x || !w || !y) return fail(BV_ERR_ARG, "bv_conv_transpose1d_ws: null pointer");
  if (B < 1 || Cin < 1 || T < 1 || Cout < 1 || K < 1 || K > 64 || stride < 1 || stride > 16 ||
      pad < 0)
    return fail(BV_ERR_SHAPE, "bv_conv_transpose1d_ws: B=%d Cin=%d T=%d Cout=%d K=%d s=%d pad=%d",
                B, Cin, T, Cout, K, stride, pad);
  const long long Tout = (long long)(T - 1) * stride + K - 2LL * pad;
  if (Tout < 1 || Tout > 0x7fffffffLL)
    return fail(BV_ERR_SHAPE, "bv_conv_transpose1d_ws: output length %lld", Tout);
  const size_t nin = (size_t)B * Cin * T, nout = (size_t)B * Cout * Tout;
  const ConvTPlan plan = convt_plan(B, Cin, T, Cout, K, stride);
  if (plan.total > 0 && (!workspace || ws_bytes < plan.total))
    return fail(BV_ERR_WORKSPACE, "bv_conv_transpose1d_ws: workspace %zu bytes, need %zu",
                ws_bytes, plan.total);
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return fail(BV_ERR_ARG, "bv_conv_transpose1d_ws: workspace not 256-byte aligned");
  const float *wsf = static_cast<const float *>(workspace);
  const size_t nws = plan.total / sizeof(float);
  if (overlaps(x, nin, y, nout) || (nws && (overlaps(x, nin, wsf, nws) || overlaps(y, nout, wsf, nws))))
    return fail(BV_ERR_ARG, "bv_conv_transpose1d_ws: x, y and workspace must be disjoint");
  BV_TRY(check_device());
  cudaStream_t st = as_stream(stream);
  char *w8 = static_cast<char *>(workspace);
  if (plan.path == 2) {
    float *xhi = reinterpret_cast<float *>(w8);
    float *xlo = reinterpret_cast<float *>(w8 + plan.plane);
    float *wp = reinterpret_cast<float *>(w8 + 2 * plan.plane);
    const bool f16 = tm_f16_ok(Cin);
    BV_TRY(launch_transpose_split(x, xhi, xlo, B, Cin, T, st, f16));
    return launch_conv_transpose1d_tm(xhi, xlo, B, Cin, T, w, bias, Cout, K, stride, pad, y, wp,
                                      st, f16);
  }
  if (plan.path == 1)
    return launch_conv_transpose1d_tc(x, B, Cin, T, w, bias, Cout, K, stride, pad, y,
                                      reinterpret_cast<float *>(w8), st);
  return launch_conv_transpose1d(x, B, Cin, T, w, bias, Cout, K, stride, pad, y, st);
}

}  // extern "C"

// --------------------------------------------------------------- decoder

namespace bv {
namespace {

bv_status check_config(const bv_decoder_config *c) {
  if (!c) return fail(BV_ERR_ARG, "decoder: null config");
  if (c->in_channels < 1 || c->pre_channels < 1 || c->out_channels < 1)
    return fail(BV_ERR_SHAPE, "decoder: channel counts must be >= 1");
  if (c->pre_kernel < 1 || c->pre_kernel % 2 == 0 || c->pre_kernel > 31 || c->post_kernel < 1 ||
      c->post_kernel % 2 == 0 || c->post_kernel > 31)
    return fail(BV_ERR_SHAPE, "decoder: pre/post kernels must be odd and <= 31");
  if (c->n_up < 0 || c->n_up > BV_MAX_UP) return fail(BV_ERR_SHAPE, "decoder: n_up %d", c->n_up);
  for (int i = 0; i < c->n_up; ++i) {
    if (c->up_rate[i] < 1 || c->up_rate[i] > 16 || c->up_kernel[i] < c->up_rate[i] ||
        c->up_kernel[i] > 64 || c->up_channels[i] < 1)
      return fail(BV_ERR_SHAPE, "decoder: stage %d rate %d kernel %d channels %d", i,
                  c->up_rate[i], c->up_kernel[i], c->up_channels[i]);
  }
  if (c->n_blocks < 1 || c->n_blocks > BV_MAX_BLOCKS)
    return fail(BV_ERR_SHAPE, "decoder: n_blocks %d", c->n_blocks);
  for (int j = 0; j < c->n_blocks; ++j)
    if (c->block_kernel[j] < 1 || c->block_kernel[j] % 2 == 0 || c->block_kernel[j] > 31)
      return fail(BV_ERR_SHAPE, "decoder: block kernel %d must be odd", c->block_kernel[j]);
  if (c->n_dilations < 1 || c->n_dilations > BV_MAX_DIL)
    return fail(BV_ERR_SHAPE, "decoder: n_dilations %d", c->n_dilations);
  for (int u = 0; u < c->n_dilations; ++u)
    if (c->dilation[u] < 1) return fail(BV_ERR_SHAPE, "decoder: dilation %d", c->dilation[u]);
  if (c->final_act < 0 || c->final_act > 2) return fail(BV_ERR_ARG, "decoder: final_act %d", c->final_act);
  if (c->tile_frames < 0 || c->overlap_frames < 0 ||
      (c->tile_frames > 0 && c->overlap_frames >= c->tile_frames))
    return fail(BV_ERR_SHAPE, "decoder: tile %d overlap %d", c->tile_frames, c->overlap_frames);
  if (c->latent_channels < 0)
    return fail(BV_ERR_SHAPE, "decoder: latent_channels %d", c->latent_channels);
  if (c->tf32_only != 0 && c->tf32_only != 1)
    return fail(BV_ERR_ARG, "decoder: tf32_only %d", c->tf32_only);
  return BV_OK;
}

// Channels of the z a decode call takes: normalised latents with the front
// end, else the decoder's input.
int z_channels(const bv_decoder_config *c) {
  return c->latent_channels > 0 ? c->latent_channels : c->in_channels;
}

// The front end's output [B, in_channels, F] (nothing without a front end).
size_t front_ws(const bv_decoder_config *c, long long B, long long F) {
  return c->latent_channels > 0 ? align_up((size_t)B * c->in_channels * F * sizeof(float)) : 0;
}

long long hop_of(const bv_decoder_config *c) {
  long long h = 1;
  for (int i = 0; i < c->n_up; ++i) h *= c->up_rate[i];
  return h;
}

// Largest B*C*T over the stored layers of an untiled decode (z excluded).
long long max_elems(const bv_decoder_config *c, long long B, long long F) {
  long long n = F, m = B * c->pre_channels * F;
  for (int i = 0; i < c->n_up; ++i) {
    const int s = c->up_rate[i], k = c->up_kernel[i];
    n = (n - 1) * s + k - 2 * ((k - s) / 2);
    const long long e = B * c->up_channels[i] * n;
    if (e > m) m = e;
  }
  return m;
}

// Repacked ConvT weights for the tensor-core path (one buffer, reused by
// every stage that takes that path).
size_t convt_ws(const bv_decoder_config *c) {
  size_t m = 0;
  int C = c->pre_channels;
  for (int i = 0; i < c->n_up; ++i) {
    const int Co = c->up_channels[i], k = c->up_kernel[i], sr = c->up_rate[i];
    size_t b = 0;
    if (conv_transpose1d_tm_supported(C, Co, k, sr))
      b = conv_transpose1d_tm_workspace(C, Co, k, sr);
    else if (conv_transpose1d_tc_supported(C, Co, k, sr))
      b = conv_transpose1d_tc_workspace(C, Co, k, sr);
    if (b > m) m = b;
    C = Co;
  }
  return align_up(m);
}

// Pre-split weights of every conv the tensor-core path takes: tf32(W) then
// W - tf32(W), written once per decode call and read by every tile group.
struct DecoderSplit {
  const float *pre = nullptr, *post = nullptr;
  AmpSplit amp[BV_MAX_UP][BV_MAX_BLOCKS] = {};
};

// Walk the decoder's convs in a fixed order; f(Cin, Cout, K, src, kind, i, j,
// u, tm) is called for each conv a tensor-core path supports (src may be null
// when only sizes are wanted); tm: the AMP conv takes the time-major path.
template <class F>
void for_each_tc_conv(const bv_decoder_config *c, const bv_decoder_weights *w, F &&f) {
  if (conv1d_tc_supported(c->in_channels, c->pre_channels, c->pre_kernel, 1))
    f(c->in_channels, c->pre_channels, c->pre_kernel, w ? w->pre_w : nullptr, 0, -1, -1, -1,
      false);
  for (int i = 0; i < c->n_up; ++i) {
    const int C = c->up_channels[i];
    for (int j = 0; j < c->n_blocks; ++j) {
      const int K = c->block_kernel[j];
      for (int u = 0; u < c->n_dilations; ++u) {
        const int d = c->dilation[u];
        const bool tm1 = conv1d_tm_supported(C, C, K, d), tm2 = conv1d_tm_supported(C, C, K, 1);
        if (tm1 || conv1d_tc_supported(C, C, K, d))
          f(C, C, K, w ? w->amp[i][j].conv1_w[u] : nullptr, 1, i, j, u, tm1);
        if (tm2 || conv1d_tc_supported(C, C, K, 1))
          f(C, C, K, w ? w->amp[i][j].conv2_w[u] : nullptr, 2, i, j, u, tm2);
      }
    }
  }
  const int Cl = c->n_up > 0 ? c->up_channels[c->n_up - 1] : c->pre_channels;
  if (conv1d_tc_supported(Cl, c->out_channels, c->post_kernel, 1))
    f(Cl, c->out_channels, c->post_kernel, w ? w->post_w : nullptr, 3, -1, -1, -1, false);
}

size_t split_ws(const bv_decoder_config *c) {
  size_t s = 0;
  for_each_tc_conv(c, nullptr,
                   [&](int Cin, int Cout, int K, const float *, int, int, int, int, bool tm) {
                     s += align_up(2 * (size_t)(tm ? tm_cin_pad(Cin) : Cin) * Cout * K *
                                   sizeof(float));
                   });
  return s;
}

// Fill `out` with slots in ws (size split_ws) and launch the split kernels.
// With launch false only the slots are filled in (the weights were split into
// ws earlier, by bv_decoder_prepare).
bv_status split_weights(const bv_decoder_config *c, const bv_decoder_weights *w, char *ws,
                        DecoderSplit *out, cudaStream_t st, bool launch = true) {
  SplitTable tab;
  tab.n = 0;
  bv_status status = BV_OK;
  size_t off = 0;
  for_each_tc_conv(c, w, [&](int Cin, int Cout, int K, const float *src, int kind, int i, int j,
                             int u, bool tm) {
    if (status != BV_OK) return;
    const long long count = (long long)Cin * Cout * K;
    float *dst = reinterpret_cast<float *>(ws + off);
    off += align_up(2 * (size_t)(tm ? tm_cin_pad(Cin) : Cin) * Cout * K * sizeof(float));
    // an unaligned weight sends a [B, C, T] conv to the SIMT path: no split needed
    if (!tm && (reinterpret_cast<uintptr_t>(src) & 15u) != 0) return;
    if (kind == 0) {
      out->pre = dst;
    } else if (kind == 1) {
      out->amp[i][j].conv1[u] = dst;
      out->amp[i][j].tm1[u] = tm;
    } else if (kind == 2) {
      out->amp[i][j].conv2[u] = dst;
      out->amp[i][j].tm2[u] = tm;
    } else {
      out->post = dst;
    }
    tab.src[tab.n] = src;
    tab.dst[tab.n] = dst;
    tab.count[tab.n] = count;
    tab.cin[tab.n] = tm ? Cin : 0;
    tab.k[tab.n] = K;
    // the AMP convs' time-major operands come from the activation, in fp16
    // where tm_f16_ok unless the config asks for 3xTF32 throughout
    const bool f16 = tm && (kind == 1 || kind == 2) && tm_f16_ok(Cin) && !c->tf32_only;
    tab.f16[tab.n] = f16;
    if (kind == 1 || kind == 2) out->amp[i][j].f16 = f16;
    if (++tab.n == kMaxSplit) {
      if (launch) status = launch_split_weights(tab, st);
      tab.n = 0;
    }
  });
  if (status != BV_OK || !launch) return status;
  return launch_split_weights(tab, st);
}

// A, S, cur, h1, h2 in [B, C, T] and the two time-major planes, then the
// repacked transposed-conv weights.
// Buffers of one untiled decode, each max B C T floats: A (stage output) and S
// (ConvT output); per AMP block its scratch (cur, h1, h2 and the two
// time-major planes); for blocks 1.. their own outputs, summed into A.
int core_planes(const bv_decoder_config *c) { return 2 + 5 * c->n_blocks + (c->n_blocks - 1); }

// prepared: the transposed convs' phase weights come packed with the
// prepared weights, so no repack buffer
size_t core_ws(const bv_decoder_config *c, long long B, long long F, bool prepared = false) {
  return core_planes(c) * align_up((size_t)max_elems(c, B, F) * sizeof(float)) +
         (prepared ? 0 : convt_ws(c));
}

// Streams on which the AMP blocks of a stage run side by side (one per block),
// created once per device and kept until exit, with the events that fork them
// from and join them back to the caller's stream.  `mu` is held from the fork
// record to the last join wait of a stage, so calls from several host threads
// on one device enqueue their fork/join sequences one at a time: a stream wait
// takes the event's state at the time of the wait call, so no call can wait on
// another call's fork point.  (Their work still shares these streams.)
struct AuxStreams {
  cudaStream_t s[BV_MAX_BLOCKS];
  cudaEvent_t fork, join[BV_MAX_BLOCKS];
  std::mutex mu;
  bool ok = false;
};

AuxStreams *aux_streams() {
  static AuxStreams per_dev[32];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 32) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  AuxStreams &a = per_dev[dev];
  if (!a.ok) {
    bool good = cudaEventCreateWithFlags(&a.fork, cudaEventDisableTiming) == cudaSuccess;
    for (int j = 0; j < BV_MAX_BLOCKS && good; ++j)
      good = cudaStreamCreateWithFlags(&a.s[j], cudaStreamNonBlocking) == cudaSuccess &&
             cudaEventCreateWithFlags(&a.join[j], cudaEventDisableTiming) == cudaSuccess;
    if (!good) {
      cudaGetLastError();
      return nullptr;
    }
    a.ok = true;
  }
  return &a;
}

struct TilePlan {
  bool tiled = false;
  int step = 0, n_tiles = 1;
  int n_full = 0;   // tiles of tile_frames frames
  int last_len = 0; // frames of a shorter last tile (0: none)
};

TilePlan plan_tiles(const bv_decoder_config *c, int F) {
  TilePlan p;
  if (c->tile_frames <= 0 || c->tile_frames >= F) return p;
  p.tiled = true;
  p.step = c->tile_frames - c->overlap_frames;
  int start = 0, n = 1;
  while (start + c->tile_frames < F) {
    start += p.step;
    ++n;
  }
  p.n_tiles = n;
  const int last = F - start;
  if (last == c->tile_frames) {
    p.n_full = n;
  } else {
    p.n_full = n - 1;
    p.last_len = last;
  }
  return p;
}

// The decode as units: unit u = k B + b is tile k of side b (an untiled
// decode is one tile of all `frames`).  Full tiles come first; a shorter last
// tile, if any, is tile n_tiles - 1.
struct UnitGeom {
  int n_tiles = 1, tile_len = 0, step = 0, n_full = 1, last_len = 0;
  long long pitch = 0;  // samples per unit row: tile_len * hop
};

UnitGeom unit_geom(const bv_decoder_config *c, int F) {
  const TilePlan tp = plan_tiles(c, F);
  UnitGeom g;
  if (tp.tiled) {
    g.n_tiles = tp.n_tiles;
    g.tile_len = c->tile_frames;
    g.step = tp.step;
    g.n_full = tp.n_full;
    g.last_len = tp.last_len;
  } else {
    g.tile_len = g.step = F;
  }
  g.pitch = (long long)g.tile_len * hop_of(c);
  return g;
}

// Units [u0, u1) split into full-tile units and last-tile units.
struct UnitRange {
  long long full_u0 = 0, full_n = 0, last_u0 = 0, last_n = 0;
};

UnitRange unit_range(const UnitGeom &g, int B, long long u0, long long u1) {
  UnitRange r;
  const long long full_units = (long long)g.n_full * B;
  r.full_u0 = u0;
  r.full_n = std::max(0LL, std::min(u1, full_units) - u0);
  r.last_u0 = std::max(u0, full_units);
  r.last_n = g.last_len > 0 ? std::max(0LL, u1 - r.last_u0) : 0;
  return r;
}

// Workspace of decoding a unit range (split weights excluded): the gathered
// latents of both kinds of unit, and the core buffers of the larger decode.
size_t units_ws(const bv_decoder_config *c, const UnitGeom &g, const UnitRange &r,
                bool prepared = false) {
  size_t s = align_up((size_t)r.full_n * c->in_channels * g.tile_len * sizeof(float)) +
             align_up((size_t)r.last_n * c->in_channels * g.last_len * sizeof(float));
  size_t core = r.full_n > 0 ? core_ws(c, r.full_n, g.tile_len, prepared) : 0;
  if (r.last_n > 0) core = std::max(core, core_ws(c, r.last_n, g.last_len, prepared));
  return s + core;
}

size_t unit_rows_bytes(const bv_decoder_config *c, const UnitGeom &g, long long n_units) {
  return align_up((size_t)n_units * c->out_channels * g.pitch * sizeof(float));
}

// Workspace of a decode; with prepared weights (bv_decoder_prepare) neither
// the split weights nor the ConvT repack buffer live in it.
size_t decode_ws(const bv_decoder_config *c, int B, int F, bool prepared = false) {
  const UnitGeom g = unit_geom(c, F);
  const size_t sw = prepared ? 0 : split_ws(c);
  if (g.n_tiles == 1) return sw + front_ws(c, B, F) + core_ws(c, B, F, prepared);
  const long long n_units = (long long)g.n_tiles * B;
  return sw + front_ws(c, B, F) + unit_rows_bytes(c, g, n_units) +
         units_ws(c, g, unit_range(g, B, 0, n_units), prepared);
}

// The prepared weights: the split weights (split_ws bytes, split_weights'
// layout), then the packed phase weights of every ConvT stage that runs on a
// tensor-core kernel.
size_t prepared_convt_bytes(const bv_decoder_config *c, int i, int Cin) {
  const int Co = c->up_channels[i], k = c->up_kernel[i], sr = c->up_rate[i];
  if (conv_transpose1d_tm_supported(Cin, Co, k, sr))
    return align_up(conv_transpose1d_tm_workspace(Cin, Co, k, sr));
  if (conv_transpose1d_tc_supported(Cin, Co, k, sr))
    return align_up(conv_transpose1d_tc_workspace(Cin, Co, k, sr));
  return 0;
}

size_t prepared_ws(const bv_decoder_config *c) {
  size_t s = split_ws(c);
  int C = c->pre_channels;
  for (int i = 0; i < c->n_up; ++i) {
    s += prepared_convt_bytes(c, i, C);
    C = c->up_channels[i];
  }
  return s;
}

// Slots of the ConvT stages' packed weights in a prepared buffer (nullptr:
// the stage packs nothing).
void prepared_convt_slots(const bv_decoder_config *c, const char *base,
                          const float *out[BV_MAX_UP]) {
  size_t off = split_ws(c);
  int C = c->pre_channels;
  for (int i = 0; i < c->n_up; ++i) {
    const size_t b = prepared_convt_bytes(c, i, C);
    out[i] = b ? reinterpret_cast<const float *>(base + off) : nullptr;
    off += b;
    C = c->up_channels[i];
  }
}

// With the latent front end, z [latent_ch, B, F] -> the decoder's input in
// the workspace (advanced past it); otherwise z itself.
bv_status run_front_end(const bv_decoder_config *c, const bv_decoder_weights *w, const float *&z,
                        int B, int F, char *&ws, cudaStream_t st) {
  if (c->latent_channels <= 0) return BV_OK;
  float *zin = reinterpret_cast<float *>(ws);
  ws += front_ws(c, B, F);
  BV_TRY(launch_latent_front_end(z, c->latent_channels, B, F, w->latents_mean, w->latents_std,
                                 w->dec_in_w, w->dec_in_b, c->in_channels, zin, st));
  z = zin;
  return BV_OK;
}

bv_status check_weights(const bv_decoder_config *c, const bv_decoder_weights *w) {
  if (!w) return fail(BV_ERR_ARG, "decoder: null weights");
  if (c->latent_channels > 0 && (!w->latents_mean || !w->latents_std || !w->dec_in_w))
    return fail(BV_ERR_ARG, "decoder: null latents_mean / latents_std / dec_in_w");
  if (!w->pre_w || !w->post_w || !w->post_log_alpha || !w->post_log_beta || !w->up_filter ||
      !w->down_filter)
    return fail(BV_ERR_ARG, "decoder: null conv_pre / act_post / conv_post weight or filter");
  for (int i = 0; i < c->n_up; ++i) {
    if (!w->up_w[i]) return fail(BV_ERR_ARG, "decoder: null ups.%d weight", i);
    for (int j = 0; j < c->n_blocks; ++j) {
      const bv_amp_params &p = w->amp[i][j];
      BV_TRY(check_amp_params(&p, c->up_channels[i]));
      if (p.kernel_size != c->block_kernel[j] || p.n_dilations != c->n_dilations)
        return fail(BV_ERR_ARG, "decoder: amp[%d][%d] kernel/dilations differ from the config", i, j);
      for (int u = 0; u < c->n_dilations; ++u)
        if (p.dilation[u] != c->dilation[u])
          return fail(BV_ERR_ARG, "decoder: amp[%d][%d] dilation differs from the config", i, j);
    }
  }
  return BV_OK;
}

// One untiled decode of B rows into y rows of length F*hop, row pitch
// y_pitch samples.
// Weights prepared for a decode: split tensor-core weights and, per ConvT
// stage, its packed phase weights (nullptr: packed into the workspace).
// A decoder's transposed conv of Cin input channels takes the fp16 split
// (where the time-major kernel runs it at all).
bool convt_f16(const bv_decoder_config *c, int Cin) { return tm_f16_ok(Cin) && !c->tf32_only; }

struct DecoderPrep {
  DecoderSplit sw;
  const float *convt[BV_MAX_UP] = {};
};

bv_status decode_core(const bv_decoder_config *c, const bv_decoder_weights *w,
                      const DecoderPrep &pp, const float *z, int B, int F, float *y,
                      long long y_pitch, char *ws, cudaStream_t st) {
  const DecoderSplit &sw = pp.sw;
  const size_t sz = align_up((size_t)max_elems(c, B, F) * sizeof(float));
  auto plane = [&](int k) { return reinterpret_cast<float *>(ws + (size_t)k * sz); };
  float *A = plane(0);
  float *S = plane(1);
  const int nb = c->n_blocks;
  AmpScratch sb[BV_MAX_BLOCKS];
  float *Ab[BV_MAX_BLOCKS];  // block j's output (block 0 writes A)
  for (int j = 0; j < nb; ++j) {
    const int k = 2 + 5 * j;
    sb[j] = AmpScratch{plane(k), plane(k + 1), plane(k + 2), plane(k + 3), plane(k + 4)};
    Ab[j] = j == 0 ? A : plane(2 + 5 * nb + (j - 1));
  }
  const AmpScratch &s = sb[0];
  float *WP = plane(core_planes(c));  // repacked ConvT weights
  // The blocks of a stage are independent until their mean: they run side by
  // side on one stream each and their outputs are summed in block order.
  // With the library's per-kernel timers on they run in order on the
  // caller's stream, so that every launch's event time is its own, and
  // accumulate through the epilogue (the same sums in the same order, but the
  // epilogue fuses scale and add into one multiply-add, so the two paths can
  // differ in the last bit).
  AuxStreams *aux = (nb > 1 && !g_timing_on.load(std::memory_order_relaxed)) ? aux_streams()
                                                                              : nullptr;
  int C = c->pre_channels, n = F;
  Epi plain{nullptr, 1.0f, 0, 0};
  BV_TRY(launch_conv1d(z, B, c->in_channels, F, w->pre_w, w->pre_b, C, c->pre_kernel, 1,
                       (c->pre_kernel - 1) / 2, plain, A, F, F, st, sw.pre));
  for (int i = 0; i < c->n_up; ++i) {
    const int sr = c->up_rate[i], k = c->up_kernel[i], Co = c->up_channels[i];
    const int pad = (k - sr) / 2;
    const int n2 = (n - 1) * sr + k - 2 * pad;
    if (conv_transpose1d_tm_supported(C, Co, k, sr)) {
      // time-major: the stage input goes to block 0's operand planes first,
      // in the fp16 split where C allows and the config does not ask for
      // 3xTF32 (the prepared phase weights were packed by the same rule)
      const bool f16 = convt_f16(c, C);
      BV_TRY(launch_transpose_split(A, s.xhi, s.xlo, B, C, n, st, f16));
      if (pp.convt[i])
        BV_TRY(launch_conv_transpose1d_tm_packed(s.xhi, s.xlo, B, C, n, pp.convt[i], w->up_b[i],
                                                 Co, k, sr, pad, S, st, f16));
      else
        BV_TRY(launch_conv_transpose1d_tm(s.xhi, s.xlo, B, C, n, w->up_w[i], w->up_b[i], Co, k,
                                          sr, pad, S, WP, st, f16));
    } else if (conv_transpose1d_tc_supported(C, Co, k, sr)) {
      if (pp.convt[i])
        BV_TRY(launch_conv_transpose1d_tc_packed(A, B, C, n, pp.convt[i], w->up_b[i], Co, k, sr,
                                                 pad, S, st));
      else
        BV_TRY(launch_conv_transpose1d_tc(A, B, C, n, w->up_w[i], w->up_b[i], Co, k, sr, pad, S,
                                          WP, st));
    } else
      BV_TRY(launch_conv_transpose1d(A, B, C, n, w->up_w[i], w->up_b[i], Co, k, sr, pad, S, st));
    C = Co;
    n = n2;
    const float scale = 1.0f / (float)nb;
    if (aux) {
      std::lock_guard<std::mutex> enqueue(aux->mu);
      CUDA_TRY(cudaEventRecord(aux->fork, st));
      for (int j = 0; j < nb; ++j) CUDA_TRY(cudaStreamWaitEvent(aux->s[j], aux->fork, 0));
      for (int j = 0; j < nb; ++j)
        BV_TRY(run_amp_block(S, B, C, n, w->amp[i][j], Ab[j], scale, 0, sb[j], aux->s[j],
                             &sw.amp[i][j]));
      for (int j = 0; j < nb; ++j) {
        CUDA_TRY(cudaEventRecord(aux->join[j], aux->s[j]));
        CUDA_TRY(cudaStreamWaitEvent(st, aux->join[j], 0));
      }
      Parts parts{nb - 1, {}};
      for (int j = 1; j < nb; ++j) parts.p[j - 1] = Ab[j];
      BV_TRY(launch_add_parts(A, parts, (long long)B * C * n, st));
    } else {
      for (int j = 0; j < nb; ++j)
        BV_TRY(run_amp_block(S, B, C, n, w->amp[i][j], A, scale, j > 0, s, st, &sw.amp[i][j]));
    }
  }
  BV_TRY(launch_activation(A, s.h1, B, C, n, w->post_log_alpha, w->post_log_beta, w->up_filter,
                           w->down_filter, 1e-9f, st));
  const long long L = (long long)F * hop_of(c);
  Epi fin{nullptr, 1.0f, 0, c->final_act};
  return launch_conv1d(s.h1, B, C, n, w->post_w, w->post_b, c->out_channels, c->post_kernel, 1,
                       (c->post_kernel - 1) / 2, fin, y, (int)L, (int)y_pitch, st, sw.post);
}

// Decode units [r.full_u0, ...) into rows of y_units (unit u at row u - u0,
// out_channels x g.pitch samples each; a last-tile row holds last_len * hop).
bv_status decode_units_impl(const bv_decoder_config *c, const bv_decoder_weights *w,
                            const DecoderPrep &sw, const float *z, int B, int F,
                            const UnitGeom &g, const UnitRange &r, float *y_units, char *ws,
                            cudaStream_t st) {
  char *p = ws;
  float *zf = reinterpret_cast<float *>(p);
  p += align_up((size_t)r.full_n * c->in_channels * g.tile_len * sizeof(float));
  float *zl = reinterpret_cast<float *>(p);
  p += align_up((size_t)r.last_n * c->in_channels * g.last_len * sizeof(float));
  if (r.full_n > 0) {
    BV_TRY(launch_gather_tiles(z, zf, B, c->in_channels, F, g.step, g.tile_len, r.full_u0,
                               r.full_n, st));
    BV_TRY(decode_core(c, w, sw, zf, (int)r.full_n, g.tile_len, y_units, g.pitch, p, st));
  }
  if (r.last_n > 0) {
    BV_TRY(launch_gather_tiles(z, zl, B, c->in_channels, F, g.step, g.last_len, r.last_u0,
                               r.last_n, st));
    float *yl = y_units + (size_t)r.full_n * c->out_channels * g.pitch;
    BV_TRY(decode_core(c, w, sw, zl, (int)r.last_n, g.last_len, yl, g.pitch, p, st));
  }
  return BV_OK;
}

// The weights a decode reads: from the prepared buffer when the weights carry
// one, else split into the workspace now (advanced past them).
bv_status prepare_for_decode(const bv_decoder_config *c, const bv_decoder_weights *w, char *&ws,
                             DecoderPrep *pp, cudaStream_t st) {
  if (w->prepared) {
    char *base = const_cast<char *>(static_cast<const char *>(w->prepared));
    BV_TRY(split_weights(c, w, base, &pp->sw, st, false));
    prepared_convt_slots(c, base, pp->convt);
    return BV_OK;
  }
  BV_TRY(split_weights(c, w, ws, &pp->sw, st));
  ws += split_ws(c);
  return BV_OK;
}

// y[b, o, t] = mean over the tiles covering t of their unit rows (all
// n_tiles B units in y_units, in unit order).
bv_status stitch_units(const bv_decoder_config *c, const UnitGeom &g, int B, int F,
                       const float *y_units, float *y, cudaStream_t st) {
  const long long hop = hop_of(c);
  TileGroups tg{};
  tg.n = 0;
  if (g.n_full > 0) {
    tg.data[tg.n] = y_units;
    tg.k0[tg.n] = 0;
    tg.count[tg.n] = g.n_full;
    tg.len_samples[tg.n] = (long long)g.tile_len * hop;
    tg.pitch[tg.n] = g.pitch;
    ++tg.n;
  }
  if (g.last_len > 0) {
    tg.data[tg.n] = y_units + (size_t)g.n_full * B * c->out_channels * g.pitch;
    tg.k0[tg.n] = g.n_full;
    tg.count[tg.n] = 1;
    tg.len_samples[tg.n] = (long long)g.last_len * hop;
    tg.pitch[tg.n] = g.pitch;
    ++tg.n;
  }
  tg.max_len_samples = (long long)g.tile_len * hop;
  return launch_stitch_tiles(tg, y, B, c->out_channels, (long long)F * hop, (int)(g.step * hop),
                             st);
}

bv_status decode_impl(const bv_decoder_config *c, const bv_decoder_weights *w, const float *z,
                      int B, int F, float *y, char *ws, cudaStream_t st) {
  const UnitGeom g = unit_geom(c, F);
  DecoderPrep sw;
  BV_TRY(prepare_for_decode(c, w, ws, &sw, st));
  BV_TRY(run_front_end(c, w, z, B, F, ws, st));
  if (g.n_tiles == 1) return decode_core(c, w, sw, z, B, F, y, (long long)F * hop_of(c), ws, st);
  // every tile of every side, then the overlap average
  const long long n_units = (long long)g.n_tiles * B;
  float *yu = reinterpret_cast<float *>(ws);
  ws += unit_rows_bytes(c, g, n_units);
  BV_TRY(decode_units_impl(c, w, sw, z, B, F, g, unit_range(g, B, 0, n_units), yu, ws, st));
  return stitch_units(c, g, B, F, yu, y, st);
}

}  // namespace

// The decoder for other parts of the library (the bandwidth-extension tail).
bv_status decoder_check(const bv_decoder_config *c, const bv_decoder_weights *w) {
  BV_TRY(check_config(c));
  return check_weights(c, w);
}
size_t decoder_workspace(const bv_decoder_config *c, int B, int F) { return decode_ws(c, B, F); }
bv_status decoder_run(const bv_decoder_config *c, const bv_decoder_weights *w, const float *z,
                      int B, int F, float *y, char *ws, cudaStream_t st) {
  return decode_impl(c, w, z, B, F, y, ws, st);
}
long long decoder_hop(const bv_decoder_config *c) { return hop_of(c); }

}  // namespace bv

extern "C" {

int64_t bv_decoder_param_count(const bv_decoder_config *c) {
  if (check_config(c) != BV_OK) return -1;
  int64_t n = (int64_t)c->pre_channels * c->in_channels * c->pre_kernel + c->pre_channels;
  int64_t C = c->pre_channels;
  for (int i = 0; i < c->n_up; ++i) {
    const int64_t Co = c->up_channels[i];
    n += C * Co * c->up_kernel[i] + Co;
    for (int j = 0; j < c->n_blocks; ++j)
      n += (int64_t)c->n_dilations * (4 * Co + 2 * (Co * Co * c->block_kernel[j] + Co));
    C = Co;
  }
  n += 2 * C + (int64_t)c->out_channels * C * c->post_kernel + c->out_channels;
  return n;
}

bv_status bv_decoder_weights_from_flat(const bv_decoder_config *c, const float *flat,
                                       const float *up_filter, const float *down_filter,
                                       bv_decoder_weights *out) {
  g_err[0] = 0;
  BV_TRY(check_config(c));
  if (!flat || !up_filter || !down_filter || !out)
    return fail(BV_ERR_ARG, "bv_decoder_weights_from_flat: null pointer");
  std::memset(out, 0, sizeof(*out));
  const float *p = flat;
  auto take = [&](size_t n) {
    const float *q = p;
    p += n;
    return q;
  };
  size_t C = c->pre_channels;
  out->pre_w = take(C * c->in_channels * c->pre_kernel);
  out->pre_b = take(C);
  for (int i = 0; i < c->n_up; ++i) {
    const size_t Co = c->up_channels[i];
    out->up_w[i] = take(C * Co * c->up_kernel[i]);
    out->up_b[i] = take(Co);
    C = Co;
    for (int j = 0; j < c->n_blocks; ++j) {
      bv_amp_params &a = out->amp[i][j];
      const size_t K = c->block_kernel[j];
      a.kernel_size = (int)K;
      a.n_dilations = c->n_dilations;
      a.up_filter = up_filter;
      a.down_filter = down_filter;
      for (int u = 0; u < c->n_dilations; ++u) {
        a.dilation[u] = c->dilation[u];
        a.act_log_alpha[2 * u] = take(C);
        a.act_log_beta[2 * u] = take(C);
        a.conv1_w[u] = take(C * C * K);
        a.conv1_b[u] = take(C);
        a.act_log_alpha[2 * u + 1] = take(C);
        a.act_log_beta[2 * u + 1] = take(C);
        a.conv2_w[u] = take(C * C * K);
        a.conv2_b[u] = take(C);
      }
    }
  }
  out->post_log_alpha = take(C);
  out->post_log_beta = take(C);
  out->post_w = take((size_t)c->out_channels * C * c->post_kernel);
  out->post_b = take(c->out_channels);
  out->up_filter = up_filter;
  out->down_filter = down_filter;
  return BV_OK;
}

int64_t bv_decoder_output_length(const bv_decoder_config *c, int frames) {
  if (check_config(c) != BV_OK || frames < 1) return -1;
  return (int64_t)frames * hop_of(c);
}

size_t bv_decode_workspace_size(const bv_decoder_config *c, int B, int frames) {
  g_err[0] = 0;
  if (check_config(c) != BV_OK) return 0;
  if (B < 1 || frames < 1) {
    fail(BV_ERR_SHAPE, "bv_decode_workspace_size: B=%d frames=%d", B, frames);
    return 0;
  }
  return decode_ws(c, B, frames);
}

bv_status bv_decode(const bv_decoder_config *c, const bv_decoder_weights *w, const float *z,
                    int B, int frames, float *y, void *workspace, size_t ws_bytes,
                    void *stream) {
  g_err[0] = 0;
  BV_TRY(check_config(c));
  if (!z || !y) return fail(BV_ERR_ARG, "bv_decode: null z or y");
  if (B < 1 || frames < 1) return fail(BV_ERR_SHAPE, "bv_decode: B=%d frames=%d", B, frames);
  const long long L = (long long)frames * hop_of(c);
  if (L > 0x7fffffffLL || max_elems(c, B, frames) > (1LL << 40))
    return fail(BV_ERR_SHAPE, "bv_decode: request too large");
  BV_TRY(check_weights(c, w));
  const size_t need = decode_ws(c, B, frames, w->prepared != nullptr);
  if (!workspace || ws_bytes < need)
    return fail(BV_ERR_WORKSPACE, "bv_decode: workspace %zu bytes, need %zu", ws_bytes, need);
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return fail(BV_ERR_ARG, "bv_decode: workspace not 256-byte aligned");
  const size_t nz = (size_t)B * z_channels(c) * frames, ny = (size_t)B * c->out_channels * L;
  const float *wsf = static_cast<const float *>(workspace);
  if (overlaps(z, nz, y, ny) || overlaps(z, nz, wsf, need / 4) || overlaps(y, ny, wsf, need / 4))
    return fail(BV_ERR_ARG, "bv_decode: z, y and workspace must be disjoint");
  BV_TRY(check_device());
  return decode_impl(c, w, z, B, frames, y, static_cast<char *>(workspace), as_stream(stream));
}

bv_status bv_latent_front_end(const float *z, int C, int S, int T, const float *mean,
                              const float *std_, const float *w, const float *bias, int Cout,
                              float *out, void *stream) {
  g_err[0] = 0;
  if (!z || !mean || !std_ || !w || !out) return fail(BV_ERR_ARG, "bv_latent_front_end: null pointer");
  if (C < 1 || S < 1 || T < 1 || Cout < 1)
    return fail(BV_ERR_SHAPE, "bv_latent_front_end: C=%d S=%d T=%d Cout=%d", C, S, T, Cout);
  if (overlaps(z, (size_t)C * S * T, out, (size_t)S * Cout * T))
    return fail(BV_ERR_ARG, "bv_latent_front_end: z and out overlap");
  BV_TRY(check_device());
  return launch_latent_front_end(z, C, S, T, mean, std_, w, bias, Cout, out, as_stream(stream));
}

size_t bv_decoder_prepared_size(const bv_decoder_config *c) {
  clear_error();
  if (check_config(c) != BV_OK) return 0;
  return std::max<size_t>(prepared_ws(c), kAlign);
}

bv_status bv_decoder_prepare(const bv_decoder_config *c, const bv_decoder_weights *w,
                             void *prepared, size_t bytes, void *stream) {
  clear_error();
  BV_TRY(check_config(c));
  BV_TRY(check_weights(c, w));
  const size_t need = std::max<size_t>(prepared_ws(c), kAlign);
  if (!prepared || bytes < need)
    return fail(BV_ERR_WORKSPACE, "bv_decoder_prepare: %zu bytes, need %zu", bytes, need);
  if ((reinterpret_cast<uintptr_t>(prepared) & (kAlign - 1)) != 0)
    return fail(BV_ERR_ARG, "bv_decoder_prepare: buffer not 256-byte aligned");
  BV_TRY(check_device());
  cudaStream_t st = as_stream(stream);
  char *base = static_cast<char *>(prepared);
  DecoderSplit sw;
  BV_TRY(split_weights(c, w, base, &sw, st));
  const float *slots[BV_MAX_UP] = {};
  prepared_convt_slots(c, base, slots);
  int C = c->pre_channels;
  for (int i = 0; i < c->n_up; ++i) {
    const int Co = c->up_channels[i], k = c->up_kernel[i], sr = c->up_rate[i];
    float *wp = const_cast<float *>(slots[i]);
    if (wp && conv_transpose1d_tm_supported(C, Co, k, sr))
      BV_TRY(launch_convt_pack_tm(w->up_w[i], C, Co, k, sr, wp, st, convt_f16(c, C)));
    else if (wp)
      BV_TRY(launch_convt_pack_tc(w->up_w[i], C, Co, k, sr, wp, st));
    C = Co;
  }
  return BV_OK;
}

size_t bv_decode_workspace_size_prepared(const bv_decoder_config *c, int B, int frames) {
  clear_error();
  if (check_config(c) != BV_OK) return 0;
  if (B < 1 || frames < 1) {
    fail(BV_ERR_SHAPE, "bv_decode_workspace_size_prepared: B=%d frames=%d", B, frames);
    return 0;
  }
  return decode_ws(c, B, frames, true);
}

int bv_decoder_tile_count(const bv_decoder_config *c, int frames) {
  if (check_config(c) != BV_OK || frames < 1) return -1;
  return unit_geom(c, frames).n_tiles;
}

int64_t bv_decoder_unit_length(const bv_decoder_config *c, int frames) {
  if (check_config(c) != BV_OK || frames < 1) return -1;
  return unit_geom(c, frames).pitch;
}

size_t bv_decode_units_workspace_size(const bv_decoder_config *c, int B, int frames,
                                      int64_t unit_begin, int64_t unit_end) {
  g_err[0] = 0;
  if (check_config(c) != BV_OK) return 0;
  if (B < 1 || frames < 1) {
    fail(BV_ERR_SHAPE, "bv_decode_units_workspace_size: B=%d frames=%d", B, frames);
    return 0;
  }
  const UnitGeom g = unit_geom(c, frames);
  const long long n_units = (long long)g.n_tiles * B;
  if (unit_begin < 0 || unit_end > n_units || unit_begin >= unit_end) {
    fail(BV_ERR_SHAPE, "bv_decode_units_workspace_size: units [%lld, %lld) of %lld",
         (long long)unit_begin, (long long)unit_end, n_units);
    return 0;
  }
  return split_ws(c) + front_ws(c, B, frames) +
         units_ws(c, g, unit_range(g, B, unit_begin, unit_end));
}

bv_status bv_decode_units(const bv_decoder_config *c, const bv_decoder_weights *w, const float *z,
                          int B, int frames, int64_t unit_begin, int64_t unit_end,
                          float *y_units, void *workspace, size_t ws_bytes, void *stream) {
  g_err[0] = 0;
  BV_TRY(check_config(c));
  if (!z || !y_units) return fail(BV_ERR_ARG, "bv_decode_units: null z or y_units");
  if (B < 1 || frames < 1) return fail(BV_ERR_SHAPE, "bv_decode_units: B=%d frames=%d", B, frames);
  if ((long long)frames * hop_of(c) > 0x7fffffffLL || max_elems(c, B, frames) > (1LL << 40))
    return fail(BV_ERR_SHAPE, "bv_decode_units: request too large");
  const UnitGeom g = unit_geom(c, frames);
  const long long n_units = (long long)g.n_tiles * B;
  if (unit_begin < 0 || unit_end > n_units || unit_begin >= unit_end)
    return fail(BV_ERR_SHAPE, "bv_decode_units: units [%lld, %lld) of %lld", (long long)unit_begin,
                (long long)unit_end, n_units);
  BV_TRY(check_weights(c, w));
  const UnitRange r = unit_range(g, B, unit_begin, unit_end);
  const bool prepared = w->prepared != nullptr;
  const size_t need = (prepared ? 0 : split_ws(c)) + front_ws(c, B, frames) +
                      units_ws(c, g, r, prepared);
  if (!workspace || ws_bytes < need)
    return fail(BV_ERR_WORKSPACE, "bv_decode_units: workspace %zu bytes, need %zu", ws_bytes, need);
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return fail(BV_ERR_ARG, "bv_decode_units: workspace not 256-byte aligned");
  const size_t nz = (size_t)B * z_channels(c) * frames;
  const size_t ny = (size_t)(unit_end - unit_begin) * c->out_channels * g.pitch;
  const float *wsf = static_cast<const float *>(workspace);
  if (overlaps(z, nz, y_units, ny) || overlaps(z, nz, wsf, need / 4) ||
      overlaps(y_units, ny, wsf, need / 4))
    return fail(BV_ERR_ARG, "bv_decode_units: z, y_units and workspace must be disjoint");
  BV_TRY(check_device());
  cudaStream_t st = as_stream(stream);
  char *ws = static_cast<char *>(workspace);
  DecoderPrep sw;
  BV_TRY(prepare_for_decode(c, w, ws, &sw, st));
  BV_TRY(run_front_end(c, w, z, B, frames, ws, st));
  return decode_units_impl(c, w, sw, z, B, frames, g, r, y_units, ws, st);
}

bv_status bv_stitch_units(const bv_decoder_config *c, int B, int frames, const float *y_units,
                          float *y, void *stream) {
  g_err[0] = 0;
  BV_TRY(check_config(c));
  if (!y_units || !y) return fail(BV_ERR_ARG, "bv_stitch_units: null y_units or y");
  if (B < 1 || frames < 1) return fail(BV_ERR_SHAPE, "bv_stitch_units: B=%d frames=%d", B, frames);
  const UnitGeom g = unit_geom(c, frames);
  const long long L = (long long)frames * hop_of(c);
  if (L > 0x7fffffffLL) return fail(BV_ERR_SHAPE, "bv_stitch_units: request too large");
  const size_t nu = (size_t)g.n_tiles * B * c->out_channels * g.pitch;
  const size_t ny = (size_t)B * c->out_channels * L;
  if (overlaps(y_units, nu, y, ny)) return fail(BV_ERR_ARG, "bv_stitch_units: y_units and y overlap");
  BV_TRY(check_device());
  return stitch_units(c, g, B, frames, y_units, y, as_stream(stream));
}

size_t bv_decode_host_workspace_size(const bv_decoder_config *c, int B, int frames) {
  const size_t core = bv_decode_workspace_size(c, B, frames);
  if (core == 0) return 0;
  const long long L = (long long)frames * hop_of(c);
  return core + align_up((size_t)B * z_channels(c) * frames * sizeof(float)) +
         align_up((size_t)B * c->out_channels * L * sizeof(float));
}

bv_status bv_decode_host(const bv_decoder_config *c, const bv_decoder_weights *w,
                         const float *z_host, int B, int frames, float *y_host, void *workspace,
                         size_t ws_bytes, void *stream) {
  g_err[0] = 0;
  BV_TRY(check_config(c));
  if (!z_host || !y_host) return fail(BV_ERR_ARG, "bv_decode_host: null z or y");
  if (B < 1 || frames < 1) return fail(BV_ERR_SHAPE, "bv_decode_host: B=%d frames=%d", B, frames);
  const size_t need = bv_decode_host_workspace_size(c, B, frames);
  if (!workspace || ws_bytes < need)
    return fail(BV_ERR_WORKSPACE, "bv_decode_host: workspace %zu bytes, need %zu", ws_bytes, need);
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return fail(BV_ERR_ARG, "bv_decode_host: workspace not 256-byte aligned");
  BV_TRY(check_weights(c, w));
  BV_TRY(check_device());
  const long long L = (long long)frames * hop_of(c);
  const size_t zb = (size_t)B * z_channels(c) * frames * sizeof(float);
  const size_t yb = (size_t)B * c->out_channels * L * sizeof(float);
  char *p = static_cast<char *>(workspace);
  float *zd = reinterpret_cast<float *>(p);
  float *yd = reinterpret_cast<float *>(p + align_up(zb));
  char *core = p + align_up(zb) + align_up(yb);
  cudaStream_t st = as_stream(stream);
  cudaError_t e = cudaMemcpyAsync(zd, z_host, zb, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return fail(BV_ERR_CUDA, "bv_decode_host: H2D: %s", cudaGetErrorString(e));
  BV_TRY(decode_impl(c, w, zd, B, frames, yd, core, st));
  e = cudaMemcpyAsync(y_host, yd, yb, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return fail(BV_ERR_CUDA, "bv_decode_host: D2H: %s", cudaGetErrorString(e));
  return BV_OK;
}

}  // extern "C"
