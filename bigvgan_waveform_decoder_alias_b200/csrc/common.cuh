// Shared host/device helpers of libbv (error state, launch accounting).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdarg>
#include <cstdio>

#include "bv.h"

namespace bv {

// Records a message for bv_last_error() and returns `st`.
bv_status fail(bv_status st, const char *fmt, ...);

// Clears the calling thread's error message (every ABI entry does first).
void clear_error();

// BV_OK if the current device is an sm_100 part (checked once per device),
// else BV_ERR_CUDA.
bv_status require_device();

// Checks the last launch; BV_ERR_CUDA with the CUDA message on failure.
bv_status check_launch(const char *what);

// Counts kernel launches issued by the library.
void count_launch(uint64_t n = 1);

// Raises `func`'s dynamic shared-memory limit to at least `bytes` on the
// current device; remembered per (device, kernel), thread-safe.  Nothing to do
// up to 48 KB.  BV_ERR_CUDA (tagged `what`) if the driver refuses.
bv_status ensure_dynamic_smem(const void *func, size_t bytes, const char *what);

// Address of the device status word that bounded waits set when they give
// up (kernels take it as an argument); nullptr if it cannot be resolved.
int *device_status_ptr();
// Status word value of an fp16 operand plane written out of range.
constexpr int kStatusF16Range = 700;

// Polls after which the tensor-core kernels' bounded waits give up (a kernel
// argument; bv_debug_set_wait_limit changes it).
long long wait_limit();

// Per-launch event timing (bv_timing_enable).  Construct right before a
// launch and let it go out of scope right after it.
class LaunchTimer {
 public:
  LaunchTimer(cudaStream_t st, const char *cls, double flops, double bytes);
  ~LaunchTimer();
  LaunchTimer(const LaunchTimer &) = delete;
  LaunchTimer &operator=(const LaunchTimer &) = delete;

 private:
  int slot_ = -1;
  cudaStream_t st_;
};

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

// 4-byte asynchronous copy global -> shared (cp.async); when !ok nothing is
// read and the destination is zero-filled (src must still be a valid
// address).  Staging loops issue these back to back, so all of a thread's
// copies are in flight at once; cp_async_wait_all() then completes them.
__device__ __forceinline__ void cp_async4_zfill(float *dst, const float *src, bool ok) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(d), "l"(src),
               "r"(ok ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
  asm volatile("cp.async.wait_all;\n" ::: "memory");
}

// [a, a+na) and [b, b+nb) (in floats) overlap?
inline bool overlaps(const float *a, size_t na, const float *b, size_t nb) {
  const char *a0 = reinterpret_cast<const char *>(a), *b0 = reinterpret_cast<const char *>(b);
  return a0 < b0 + nb * sizeof(float) && b0 < a0 + na * sizeof(float);
}

inline bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Epilogue in device-friendly form.
struct Epi {
  const float *residual;  // may equal y
  float scale;
  int accumulate;
  int final_act;
};

// Grouped form for a thread that owns N outputs y[idx0 + e * stride]: the
// caller passes the group's biases already in registers (from shared memory),
// every value read from global memory (residual, the accumulated y) comes
// through the read-only path, and all N reads are issued before the N
// writes.  That is safe although residual and y may be one buffer: each index
// is read once, by the thread that then writes it, and what it reads was
// written by an earlier kernel.  (Measured on B200: a global load issued
// between stores to y -- a plain load, or even a read-only bias load -- waited
// a full memory round trip each, which made the output loop of a tensor-core
// conv tile several times longer than its stores.)
// epi_values computes the group's outputs into out (entries past `valid`
// undefined); epi_group also writes them.
template <int N>
__device__ __forceinline__ void epi_values(const float *v, const float (&bias)[N], const Epi &e,
                                           const float *y, size_t idx0, size_t stride, int valid,
                                           float (&out)[N]) {
  float r[N], a[N];
  if (e.residual || e.accumulate) {
#pragma unroll
    for (int q = 0; q < N; ++q) {
      r[q] = (e.residual && q < valid) ? __ldg(e.residual + idx0 + q * stride) : 0.0f;
      a[q] = (e.accumulate && q < valid) ? __ldg(y + idx0 + q * stride) : 0.0f;
    }
  } else {
#pragma unroll
    for (int q = 0; q < N; ++q) r[q] = a[q] = 0.0f;
  }
#pragma unroll
  for (int q = 0; q < N; ++q) {
    float t = (v[q] + bias[q] + r[q]) * e.scale + a[q];
    if (e.final_act == 1) t = fminf(fmaxf(t, -1.0f), 1.0f);
    else if (e.final_act == 2) t = tanhf(t);
    out[q] = t;
  }
}
template <int N>
__device__ __forceinline__ void epi_group(float *v, const float (&bias)[N], const Epi &e,
                                          float *y, size_t idx0, size_t stride, int valid) {
  float t[N];
  epi_values<N>(v, bias, e, y, idx0, stride, valid, t);
#pragma unroll
  for (int q = 0; q < N; ++q)
    if (q < valid) y[idx0 + q * stride] = t[q];
}

// Two-phase form for a thread that owns many outputs: epi_load folds in
// everything read from memory (bias, residual, the accumulated y) for all of
// them before epi_store writes any, so the loads overlap instead of each one
// waiting behind the previous store.  residual and y may be one buffer: every
// index is read and then written by the same thread only.
__device__ __forceinline__ float epi_load(float acc, float bias, const Epi &e, const float *yp,
                                          size_t idx) {
  float v = acc + bias;
  if (e.residual) v += e.residual[idx];
  v *= e.scale;
  if (e.accumulate) v += yp[idx];
  return v;
}
__device__ __forceinline__ float epi_final(float v, const Epi &e) {
  if (e.final_act == 1) v = fminf(fmaxf(v, -1.0f), 1.0f);
  else if (e.final_act == 2) v = tanhf(v);
  return v;
}
__device__ __forceinline__ float apply_epilogue(float acc, float bias, const Epi &e,
                                                const float *yp, size_t idx) {
  float v = acc + bias;
  if (e.residual) v += e.residual[idx];  // may alias y: plain load
  v *= e.scale;
  if (e.accumulate) v += yp[idx];
  if (e.final_act == 1) v = fminf(fmaxf(v, -1.0f), 1.0f);
  else if (e.final_act == 2) v = tanhf(v);
  return v;
}

// ---- launchers shared by the ABI and the decoder orchestration -------------

// Alias-free activation over rows (b, c) of length T.
bv_status launch_activation(const float *x, float *y, int B, int C, int T, const float *la,
                            const float *lb, const float *fu, const float *fd, float eps,
                            cudaStream_t st);

// The activation writing the time-major tensor-core conv's operand planes
// hi[b, t, c] = tf32(y), lo = y - hi instead of y [B, C, T] (C a multiple of 8;
// planes 16-byte aligned).  With f16 the planes hold fp16 values instead:
// hi = fp16(y), lo = fp16(y - hi), [B, T, C] halves at the same addresses.
bool activation_tm_supported(int C);
bv_status launch_activation_tm(const float *x, float *hi, float *lo, int B, int C, int T,
                               const float *la, const float *lb, const float *fu, const float *fd,
                               float eps, cudaStream_t st, bool f16 = false);

// Latent front end: z [C, S, T] -> out [S, Cout, T], de-normalised then
// projected by a one-tap conv w [Cout, C, 1] (+ bias or NULL).
bv_status launch_latent_front_end(const float *z, int C, int S, int T, const float *mean,
                                  const float *stdv, const float *w, const float *bias, int Cout,
                                  float *out, cudaStream_t st);

// The whole decoder (bv_decode without its argument checks): config and
// weights check, workspace bytes, run (z, y device; ws 256-byte aligned),
// samples per latent frame.
bv_status decoder_check(const bv_decoder_config *c, const bv_decoder_weights *w);
size_t decoder_workspace(const bv_decoder_config *c, int B, int F);
bv_status decoder_run(const bv_decoder_config *c, const bv_decoder_weights *w, const float *z,
                      int B, int F, float *y, char *ws, cudaStream_t st);
long long decoder_hop(const bv_decoder_config *c);

// The activation's sin^2, elementwise (for accuracy tests).
bv_status launch_sin_squared(const float *z, float *out, long long n, cudaStream_t st);

// Conv1d; writes y rows of length y_len (<= Tout: the first y_len outputs),
// row pitch y_pitch floats.
bv_status launch_conv1d(const float *x, int B, int Cin, int T, const float *w, const float *bias,
                        int Cout, int K, int dil, int pad, const Epi &ep, float *y, int y_len,
                        int y_pitch, cudaStream_t st, const float *w_split = nullptr);

// Conv1d on the tensor cores (tcgen05, 3xTF32); supported() says whether the
// shape qualifies (launch_conv1d picks it automatically).
#define BV_TRY(expr)            \
  do {                          \
    bv_status _s = (expr);      \
    if (_s != BV_OK) return _s; \
  } while (0)
#define CUDA_TRY(expr)                                                               \
  do {                                                                               \
    cudaError_t _e = (expr);                                                         \
    if (_e != cudaSuccess) return fail(BV_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(_e)); \
  } while (0)

// w_split: tf32(W) followed by W - tf32(W), each in w's layout (written by
// launch_split_weights), or nullptr, in which case the kernel splits w itself.
bool conv1d_tc_supported(int Cin, int Cout, int K, int dil);
bv_status launch_conv1d_tc(const float *x, int B, int Cin, int T, const float *w,
                           const float *w_split, const float *bias, int Cout, int K, int dil,
                           int pad, const Epi &ep, float *y, int y_len, int y_pitch,
                           cudaStream_t st);

// tf32(W) and W - tf32(W) of a batch of weight tensors in one launch: entry e
// writes dst[e][0, count) = tf32(src[e]) and dst[e][count, 2 count) = the rest.
constexpr int kMaxSplit = 96;  // keeps the table under 4 KB of kernel parameters
struct SplitTable {
  int n;
  const float *src[kMaxSplit];
  float *dst[kMaxSplit];
  long long count[kMaxSplit];
  // tap-major entries: src is [rows][cin][k] and dst[o][j cin + i] = src[o][i][j];
  // cin = 0 keeps src's order
  int cin[kMaxSplit], k[kMaxSplit];
  // tap-major entries in fp16 (tm_f16_split): hi = fp16(s W), lo = fp16(s W - hi)
  // with s = kTmF16WScale, rows padded to tm_cin_pad_f16(cin) channels per tap
  unsigned char f16[kMaxSplit];
};
bv_status launch_split_weights(const SplitTable &tab, cudaStream_t st);

// Narrow conv on the FP32 pipe (at most 32 input and output channels, at
// least 4 output channels); arguments as launch_conv1d.
bool conv1d_small_supported(int Cin, int Cout, int K, int dil);
bv_status launch_conv1d_small(const float *x, int B, int Cin, int T, const float *w,
                              const float *bias, int Cout, int K, int dil, int pad,
                              const Epi &ep, float *y, int y_len, int y_pitch, cudaStream_t st);

// acc += parts[0] + parts[1] + ... (n floats each), added in that order.
constexpr int kMaxParts = 3;
struct Parts {
  int n;
  const float *p[kMaxParts];
};
bv_status launch_add_parts(float *acc, const Parts &parts, long long n, cudaStream_t st);

// Time-major tensor-core conv: x_hi / x_lo are [B, T, Cin] planes with
// x = x_hi + x_lo, x_hi = tf32(x) (launch_transpose_split writes them);
// w_split holds tf32(W') then W' - tf32(W') for the tap-major weight matrix
// W'[o, j Cp + i] = w[o, i, j], Cp = tm_cin_pad(Cin), zero for i >= Cin
// (launch_split_weights with cin set).
// Output and epilogue as launch_conv1d ([B, Cout, y_pitch]).
bool conv1d_tm_supported(int Cin, int Cout, int K, int dil);
// Channels per tap in the time-major conv's weight rows: Cin rounded up to
// whole 32-channel blocks (the padding is zero).
__host__ __device__ constexpr int tm_cin_pad(int cin) { return (cin + 31) / 32 * 32; }
// The fp16 form of the time-major conv (f16 below): operands split into two
// fp16 parts (x = hi + lo, W scaled by kTmF16WScale into fp16's normal range,
// the products accumulated in fp32 and scaled back), 64-channel blocks (a
// 128-byte fp16 row, the geometry of a 32-channel tf32 row).  Its split
// weights take at most the bytes of the tf32 split.
constexpr float kTmF16WScale = 4096.0f;
__host__ __device__ constexpr int tm_cin_pad_f16(int cin) { return (cin + 63) / 64 * 64; }
// The time-major convs fed by the time-major activation run in fp16 when
// Cin allows: rows of 16 bytes and at most a third of padding in the blocks.
bool tm_f16_ok(int Cin);
bv_status launch_conv1d_tm(const float *x_hi, const float *x_lo, int B, int Cin, int T,
                           const float *w_split, const float *bias, int Cout, int K, int dil,
                           int pad, const Epi &ep, float *y, int y_len, int y_pitch,
                           cudaStream_t st, bool f16 = false);

// Transposed conv on the time-major kernel: x_hi / x_lo [B, T, Cin] planes
// (launch_transpose_split), each of the S output phases an ceil(K/S)-tap conv
// over the input samples with its weights repacked tap-major into wp
// (conv_transpose1d_tm_workspace bytes).  f16: planes and phase weights in
// the fp16 split (tm_f16_ok(Cin)), as launch_conv1d_tm.
bool conv_transpose1d_tm_supported(int Cin, int Cout, int K, int S);
size_t conv_transpose1d_tm_workspace(int Cin, int Cout, int K, int S);
bv_status launch_conv_transpose1d_tm(const float *x_hi, const float *x_lo, int B, int Cin, int T,
                                     const float *w, const float *bias, int Cout, int K, int S,
                                     int pad, float *y, float *wp, cudaStream_t st,
                                     bool f16 = false);

// The same with the phase weights packed beforehand (launch_convt_pack_tm
// writes at most conv_transpose1d_tm_workspace bytes, in the same split).
bv_status launch_convt_pack_tm(const float *w, int Cin, int Cout, int K, int S, float *wp,
                               cudaStream_t st, bool f16 = false);
bv_status launch_conv_transpose1d_tm_packed(const float *x_hi, const float *x_lo, int B, int Cin,
                                            int T, const float *wp, const float *bias, int Cout,
                                            int K, int S, int pad, float *y, cudaStream_t st,
                                            bool f16 = false);

// [B, C, T] -> time-major planes hi[b, t, c] = tf32(x[b, c, t]),
// lo = x - hi (f16: fp16(x) and fp16(x - hi), halves at the same addresses).
bv_status launch_transpose_split(const float *x, float *hi, float *lo, int B, int C, int T,
                                 cudaStream_t st, bool f16 = false);

// ConvTranspose1d on the tensor cores: each output phase is an ordinary conv
// over the input samples with repacked weights (wp: workspace of
// conv_transpose1d_tc_workspace bytes, rewritten by every call).
bool conv_transpose1d_tc_supported(int Cin, int Cout, int K, int S);
size_t conv_transpose1d_tc_workspace(int Cin, int Cout, int K, int S);
bv_status launch_conv_transpose1d_tc(const float *x, int B, int Cin, int T, const float *w,
                                     const float *bias, int Cout, int K, int S, int pad, float *y,
                                     float *wp, cudaStream_t st);

// Narrow ConvTranspose1d on the FP32 pipe (at most 64 input and 32 output
// channels, stride 1 or 2, at most 4 taps per phase).
bool conv_transpose1d_small_supported(int Cin, int Cout, int K, int S);
bv_status launch_conv_transpose1d_small(const float *x, int B, int Cin, int T, const float *w,
                                        const float *bias, int Cout, int K, int S, int pad,
                                        float *y, cudaStream_t st);

// The [B, C, T] tensor-core ConvT with its phase weights packed beforehand
// (launch_convt_pack_tc writes conv_transpose1d_tc_workspace bytes).
bv_status launch_convt_pack_tc(const float *w, int Cin, int Cout, int K, int S, float *wp,
                               cudaStream_t st);
bv_status launch_conv_transpose1d_tc_packed(const float *x, int B, int Cin, int T,
                                            const float *wp, const float *bias, int Cout, int K,
                                            int S, int pad, float *y, cudaStream_t st);

// ConvTranspose1d.
bv_status launch_conv_transpose1d(const float *x, int B, int Cin, int T, const float *w,
                                  const float *bias, int Cout, int K, int stride, int pad,
                                  float *y, cudaStream_t st);

}  // namespace bv
