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
// of one (input channel, tap) are contiguous, then each thread accumulates 2
// outputs x COUT channels in registers: per (i, j), two reads of x and COUT/4
// broadcast 16-byte reads of w feed 2 COUT FMAs.
#include "common.cuh"

namespace bv {
namespace {

constexpr int SM_T = 512;       // outputs per CTA
constexpr int SM_THREADS = 256;  // 2 consecutive outputs each
constexpr int SM_MAX_C = 32;

template <int COUT>  // output channels rounded up to a multiple of 4
__global__ void __launch_bounds__(SM_THREADS, 2)
conv1d_small_kernel(const float *__restrict__ x, const float *__restrict__ w,
                    const float *__restrict__ bias, float *y, int Cin, int T, int Cout, int K,
                    int dil, int pad, int y_len, int y_pitch, Epi ep) {
  static_assert(COUT % 4 == 0 && COUT <= SM_MAX_C, "output channels");
  extern __shared__ __align__(16) float sm[];
  const int halo = (K - 1) * dil;
  const int XW = (SM_T + halo + 3) & ~3;  // staged row width
  float *ws = sm;                          // [Cin K][COUT]
  float *xs = sm + Cin * K * COUT;         // [Cin][XW]
  __shared__ float bias_s[COUT];
  const int t0 = blockIdx.x * SM_T, b = blockIdx.y;
  const int tid = threadIdx.x;

  for (int idx = tid; idx < Cin * K * COUT; idx += SM_THREADS) {
    const int o = idx % COUT, ij = idx / COUT;
    const int i = ij / K, j = ij - i * K;
    ws[idx] = o < Cout ? __ldg(w + ((size_t)o * Cin + i) * K + j) : 0.0f;
  }
  const float *xb = x + (size_t)b * Cin * T;
  for (int idx = tid; idx < Cin * XW; idx += SM_THREADS) {
    const int i = idx / XW, n = idx - i * XW;
    const int t = t0 - pad + n;
    xs[idx] = (t >= 0 && t < T && n < SM_T + halo) ? __ldg(xb + (size_t)i * T + t) : 0.0f;
  }
  if (tid < COUT) bias_s[tid] = (bias && tid < Cout) ? __ldg(bias + tid) : 0.0f;
  __syncthreads();

  const int tl = 2 * tid;  // this thread's outputs t0 + tl, t0 + tl + 1
  float acc[COUT][2];
#pragma unroll
  for (int o = 0; o < COUT; ++o) acc[o][0] = acc[o][1] = 0.0f;
  for (int i = 0; i < Cin; ++i) {
    const float *xr = xs + i * XW + tl;
    const float4 *wr = reinterpret_cast<const float4 *>(ws + i * K * COUT);
    for (int j = 0; j < K; ++j) {
      const float x0 = xr[j * dil], x1 = xr[j * dil + 1];
      const float4 *wj = wr + j * (COUT / 4);
#pragma unroll
      for (int o4 = 0; o4 < COUT / 4; ++o4) {
        const float4 wv = wj[o4];
        acc[4 * o4][0] = fmaf(wv.x, x0, acc[4 * o4][0]);
        acc[4 * o4][1] = fmaf(wv.x, x1, acc[4 * o4][1]);
        acc[4 * o4 + 1][0] = fmaf(wv.y, x0, acc[4 * o4 + 1][0]);
        acc[4 * o4 + 1][1] = fmaf(wv.y, x1, acc[4 * o4 + 1][1]);
        acc[4 * o4 + 2][0] = fmaf(wv.z, x0, acc[4 * o4 + 2][0]);
        acc[4 * o4 + 2][1] = fmaf(wv.z, x1, acc[4 * o4 + 2][1]);
        acc[4 * o4 + 3][0] = fmaf(wv.w, x0, acc[4 * o4 + 3][0]);
        acc[4 * o4 + 3][1] = fmaf(wv.w, x1, acc[4 * o4 + 3][1]);
      }
    }
  }

  // epilogue, 8 channels at a time: every read (residual, accumulated y,
  // through the read-only path: each index is read once, by this thread,
  // before it writes it) ahead of the group's writes
  const int t = t0 + tl;
  if (t >= y_len) return;
  const bool two = t + 1 < y_len;
  const bool vec = two && ((((size_t)b * Cout) * y_pitch + t) % 2 == 0) && (y_pitch % 2 == 0) &&
                   ((reinterpret_cast<uintptr_t>(y) & 7u) == 0);
#pragma unroll
  for (int g = 0; g < COUT; g += 8) {
    float r[8][2], a[8][2];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int o = g + q;
      const size_t idx = ((size_t)b * Cout + o) * y_pitch + t;
      const bool ok = o < Cout;
      r[q][0] = (ok && ep.residual) ? __ldg(ep.residual + idx) : 0.0f;
      r[q][1] = (ok && two && ep.residual) ? __ldg(ep.residual + idx + 1) : 0.0f;
      a[q][0] = (ok && ep.accumulate) ? __ldg(y + idx) : 0.0f;
      a[q][1] = (ok && two && ep.accumulate) ? __ldg(y + idx + 1) : 0.0f;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int o = g + q;
      if (o < Cout) {
        const size_t idx = ((size_t)b * Cout + o) * y_pitch + t;
        const float v0 = epi_final((acc[o][0] + bias_s[o] + r[q][0]) * ep.scale + a[q][0], ep);
        const float v1 = epi_final((acc[o][1] + bias_s[o] + r[q][1]) * ep.scale + a[q][1], ep);
        if (vec) {
          *reinterpret_cast<float2 *>(y + idx) = make_float2(v0, v1);
        } else {
          y[idx] = v0;
          if (two) y[idx + 1] = v1;
        }
      }
    }
  }
}

template <int COUT>
bv_status run_small(const float *x, int B, int Cin, int T, const float *w, const float *bias,
                    int Cout, int K, int dil, int pad, const Epi &ep, float *y, int y_len,
                    int y_pitch, cudaStream_t st) {
  const int XW = (SM_T + (K - 1) * dil + 3) & ~3;
  const size_t smem = ((size_t)Cin * K * COUT + (size_t)Cin * XW) * sizeof(float);
  if (smem > 200 * 1024) return fail(BV_ERR_UNSUPPORTED, "conv1d_small: tile too large");
  static size_t configured = 0;
  if (smem > 48 * 1024 && smem > configured) {
    if (cudaFuncSetAttribute(conv1d_small_kernel<COUT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return check_launch("conv1d_small smem attribute");
    configured = smem;
  }
  dim3 grid((y_len + SM_T - 1) / SM_T, B);
  if (grid.y > 65535) return fail(BV_ERR_SHAPE, "conv1d_small: grid too large");
  {
    const double outs = (double)B * Cout * y_len;
    LaunchTimer tm(st, "conv1d_small", 2.0 * outs * Cin * K,
                   4.0 * ((double)B * Cin * T + (double)Cout * Cin * K +
                          outs * (1 + (ep.residual ? 1 : 0) + ep.accumulate)));
    conv1d_small_kernel<COUT><<<grid, SM_THREADS, smem, st>>>(x, w, bias, y, Cin, T, Cout, K, dil,
                                                              pad, y_len, y_pitch, ep);
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
#define BV_SMALL(N)                                                                           \
  if (Cout <= N)                                                                              \
    return run_small<N>(x, B, Cin, T, w, bias, Cout, K, dil, pad, ep, y, y_len, y_pitch, st);
  BV_SMALL(8)
  BV_SMALL(12)
  BV_SMALL(16)
  BV_SMALL(24)
  BV_SMALL(32)
#undef BV_SMALL
  return fail(BV_ERR_UNSUPPORTED, "conv1d_small: Cout %d", Cout);
}

}  // namespace bv
