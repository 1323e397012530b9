// Dilated Conv1d for narrow layers (at most 32 input and 32 output channels)
// on the FP32 pipe, with the bias / residual / scale / accumulate / final-op
// epilogue fused:
//
//   y[b,o,t] = bias[o] + sum_i sum_j w[o,i,j] x[b,i,t + j d - pad]
// (docs.rs cortiq-engine audiovae.rs `Conv1d::apply`; ltxaudio.rs
// `Conv1d::forward`).
//
// The decoder's last stages have 12-32 channels over hundreds of thousands of
// samples: per output only Cin K multiply-adds, so a GEMM tiling wastes most
// of its channel tile.  Here a CTA takes SM_T consecutive outputs of one batch
// row for every output channel.  It stages the input rows it needs (zero
// outside [0, T)) and all the weights, reordered so that the output channels
// of one (input channel, tap) are contiguous, then each thread accumulates 4
// consecutive outputs x COUT channels in registers: per (i, j), four reads of
// x and COUT/4 broadcast 16-byte reads of w feed 4 COUT FMAs, issued as
// packed pairs over output channels (2p, 2p + 1) against x duplicated into
// both halves: each half is an ordinary round-to-nearest FMA, so the results
// are those of scalar FMAs, in half the instructions.  The common kernel
// sizes are template arguments, so the tap loop unrolls.
#include "common.cuh"

namespace bv {
namespace {

constexpr int SM_T = 512;        // outputs per CTA
constexpr int SM_PER = 4;        // consecutive outputs per thread
constexpr int SM_THREADS = SM_T / SM_PER;
constexpr int SM_MAX_C = 32;

// COUT: output channels rounded up to a multiple of 4; KT: the kernel size
// when fixed at compile time, 0 for a runtime K
template <int COUT, int KT>
__global__ void __launch_bounds__(SM_THREADS, COUT > 24 ? 2 : 3)
conv1d_small_kernel(const float *__restrict__ x, const float *__restrict__ w,
                    const float *__restrict__ bias, float *y, int Cin, int T, int Cout, int Kr,
                    int dil, int pad, int y_len, int y_pitch, Epi ep) {
  static_assert(COUT % 4 == 0 && COUT <= SM_MAX_C, "output channels");
  const int K = KT > 0 ? KT : Kr;
  extern __shared__ __align__(16) float sm[];
  const int halo = (K - 1) * dil;
  const int XW = (SM_T + halo + 3) & ~3;  // staged row width
  float *ws = sm;                          // [Cin K][COUT]
  float *xs = sm + Cin * K * COUT;         // [Cin][XW]
  __shared__ float bias_s[COUT];
  const int t0 = blockIdx.x * SM_T, b = blockIdx.y;
  const int tid = threadIdx.x;

  // staging through cp.async, zero-filled where nothing is read: every copy
  // of the thread is in flight at once instead of one load latency each
  for (int idx = tid; idx < Cin * K * COUT; idx += SM_THREADS) {
    const int o = idx % COUT, ij = idx / COUT;
    const int i = ij / K, j = ij - i * K;
    const bool ok = o < Cout;
    cp_async4_zfill(ws + idx, ok ? w + ((size_t)o * Cin + i) * K + j : w, ok);
  }
  const float *xb = x + (size_t)b * Cin * T;
  for (int idx = tid; idx < Cin * XW; idx += SM_THREADS) {
    const int i = idx / XW, n = idx - i * XW;
    const int t = t0 - pad + n;
    const bool ok = t >= 0 && t < T && n < SM_T + halo;
    cp_async4_zfill(xs + idx, ok ? xb + (size_t)i * T + t : xb, ok);
  }
  if (tid < COUT) bias_s[tid] = (bias && tid < Cout) ? __ldg(bias + tid) : 0.0f;
  cp_async_wait_all();
  __syncthreads();

  const int tl = SM_PER * tid;  // this thread's outputs t0 + tl .. t0 + tl + SM_PER - 1
  float2 acc2[COUT / 2][SM_PER];  // output channels (2p, 2p + 1)
#pragma unroll
  for (int o = 0; o < COUT / 2; ++o)
#pragma unroll
    for (int e = 0; e < SM_PER; ++e) acc2[o][e] = make_float2(0.0f, 0.0f);
  for (int i = 0; i < Cin; ++i) {
    const float *xr = xs + i * XW + tl;
    const float4 *wr = reinterpret_cast<const float4 *>(ws + i * K * COUT);
#pragma unroll(KT > 0 ? KT : 1)
    for (int j = 0; j < K; ++j) {
      float xv[SM_PER];
#pragma unroll
      for (int e = 0; e < SM_PER; ++e) xv[e] = xr[j * dil + e];
      const float4 *wj = wr + j * (COUT / 4);
      float2 xx[SM_PER];
#pragma unroll
      for (int e = 0; e < SM_PER; ++e) xx[e] = make_float2(xv[e], xv[e]);
#pragma unroll
      for (int o4 = 0; o4 < COUT / 4; ++o4) {
        const float4 wv = wj[o4];
        const float2 w01 = make_float2(wv.x, wv.y), w23 = make_float2(wv.z, wv.w);
#pragma unroll
        for (int e = 0; e < SM_PER; ++e) {
          acc2[2 * o4][e] = __ffma2_rn(w01, xx[e], acc2[2 * o4][e]);
          acc2[2 * o4 + 1][e] = __ffma2_rn(w23, xx[e], acc2[2 * o4 + 1][e]);
        }
      }
    }
  }

  // epilogue, 4 channels at a time: every read (residual, accumulated y,
  // through the read-only path: each index is read once, by this thread,
  // before it writes it) ahead of the group's writes
  const int t = t0 + tl;
  if (t >= y_len) return;
  const int n_out = y_len - t < SM_PER ? y_len - t : SM_PER;
  const bool vec = n_out == SM_PER && (y_pitch % 4 == 0) &&
                   ((reinterpret_cast<uintptr_t>(y) & 15u) == 0);  // t is a multiple of 4
#pragma unroll
  for (int g = 0; g < COUT; g += 4) {
    float r[4][SM_PER], a[4][SM_PER];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int o = g + q;
      const size_t idx = ((size_t)b * Cout + o) * y_pitch + t;
#pragma unroll
      for (int e = 0; e < SM_PER; ++e) {
        const bool ok = o < Cout && e < n_out;
        r[q][e] = (ok && ep.residual) ? __ldg(ep.residual + idx + e) : 0.0f;
        a[q][e] = (ok && ep.accumulate) ? __ldg(y + idx + e) : 0.0f;
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int o = g + q;
      if (o < Cout) {
        const size_t idx = ((size_t)b * Cout + o) * y_pitch + t;
        float v[SM_PER];
#pragma unroll
        for (int e = 0; e < SM_PER; ++e)
          v[e] = epi_final(((o & 1 ? acc2[o >> 1][e].y : acc2[o >> 1][e].x) + bias_s[o] + r[q][e]) *
                               ep.scale + a[q][e], ep);
        if (vec) {
          *reinterpret_cast<float4 *>(y + idx) = make_float4(v[0], v[1], v[2], v[3]);
        } else {
#pragma unroll
          for (int e = 0; e < SM_PER; ++e)
            if (e < n_out) y[idx + e] = v[e];
        }
      }
    }
  }
}

template <int COUT, int KT>
bv_status run_small(const float *x, int B, int Cin, int T, const float *w, const float *bias,
                    int Cout, int K, int dil, int pad, const Epi &ep, float *y, int y_len,
                    int y_pitch, cudaStream_t st) {
  const int XW = (SM_T + (K - 1) * dil + 3) & ~3;
  const size_t smem = ((size_t)Cin * K * COUT + (size_t)Cin * XW) * sizeof(float);
  if (smem > 200 * 1024) return fail(BV_ERR_UNSUPPORTED, "conv1d_small: tile too large");
  BV_TRY(ensure_dynamic_smem((const void *)conv1d_small_kernel<COUT, KT>, smem,
                             "conv1d_small smem attribute"));
  dim3 grid((y_len + SM_T - 1) / SM_T, B);
  if (grid.y > 65535) return fail(BV_ERR_SHAPE, "conv1d_small: grid too large");
  {
    const double outs = (double)B * Cout * y_len;
    LaunchTimer tm(st, "conv1d_small", 2.0 * outs * Cin * K,
                   4.0 * ((double)B * Cin * T + (double)Cout * Cin * K +
                          outs * (1 + (ep.residual ? 1 : 0) + ep.accumulate)));
    conv1d_small_kernel<COUT, KT><<<grid, SM_THREADS, smem, st>>>(x, w, bias, y, Cin, T, Cout, K,
                                                                  dil, pad, y_len, y_pitch, ep);
  }
  count_launch();
  return check_launch("conv1d_small_kernel");
}

}  // namespace

bool conv1d_small_supported(int Cin, int Cout, int K, int dil) {
  return Cin >= 1 && Cin <= SM_MAX_C && Cout >= 4 && Cout <= SM_MAX_C && K >= 1 && K <= 32 &&
         dil >= 1 && (K - 1) * dil <= 64;
}

bv_status launch_conv1d_small(const float *x, int B, int Cin, int T, const float *w,
                              const float *bias, int Cout, int K, int dil, int pad,
                              const Epi &ep, float *y, int y_len, int y_pitch, cudaStream_t st) {
  if (B <= 0 || y_len <= 0) return BV_OK;
  if (!conv1d_small_supported(Cin, Cout, K, dil))
    return fail(BV_ERR_UNSUPPORTED, "conv1d_small: Cin %d Cout %d", Cin, Cout);
#define BV_SMALL_K(N, KK)                                                                     \
  if (K == KK)                                                                                \
    return run_small<N, KK>(x, B, Cin, T, w, bias, Cout, K, dil, pad, ep, y, y_len, y_pitch, st);
#define BV_SMALL(N)                                                                           \
  if (Cout <= N) {                                                                            \
    BV_SMALL_K(N, 3)                                                                          \
    BV_SMALL_K(N, 7)                                                                          \
    BV_SMALL_K(N, 11)                                                                         \
    return run_small<N, 0>(x, B, Cin, T, w, bias, Cout, K, dil, pad, ep, y, y_len, y_pitch, st); \
  }
  BV_SMALL(8)
  BV_SMALL(12)
  BV_SMALL(16)
  BV_SMALL(24)
  BV_SMALL(32)
#undef BV_SMALL
#undef BV_SMALL_K
  return fail(BV_ERR_UNSUPPORTED, "conv1d_small: Cout %d", Cout);
}

}  // namespace bv
