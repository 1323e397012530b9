// Dilated Conv1d as an implicit GEMM on the FP32 pipe (SIMT), with the
// bias / residual / scale / accumulate / final-activation epilogue fused.
//
//   y[b,o,t] = bias[o] + sum_i sum_j w[o,i,j] x[b,i,t + j d - pad]
// (docs.rs cortiq-engine audiovae.rs `Conv1d::apply`; ltxaudio.rs
// `Conv1d::forward`).  GEMM view: M = Cout, N = time, K = Cin * taps.
//
// A CTA owns a BM x BN output tile.  Per chunk of CK input channels it stages
// the weights w[o0.., i0.., :] (as [ci][j][m], M contiguous) and the input
// rows x[b, i0.., t0 - pad .. t0 + BN + (K-1) d - pad) once -- every tap reads
// the same staged row at offset j*d -- then each thread accumulates a
// TM x TN register tile.  A thread's TN outputs are strided by the number of
// thread columns, so a warp's shared-memory reads are consecutive.
#include "common.cuh"

namespace bv {
namespace {

template <int BM, int BN, int TM, int TN, int CK>
struct ConvCfg {
  static constexpr int NTY = BM / TM;
  static constexpr int NTX = BN / TN;
  static constexpr int THREADS = NTX * NTY;
  static constexpr int WS_PITCH = BM + 4;  // floats per (ci, j) weight row in smem
  // staged input rows [CK][W], rounded up so the weights that follow start
  // on a 16-byte boundary (they are read as float4)
  __host__ __device__ static constexpr int xs_floats(int W) { return (CK * W + 3) & ~3; }
  static size_t smem_bytes(int K, int dil) {
    const int W = BN + (K - 1) * dil;
    return ((size_t)xs_floats(W) + (size_t)CK * K * WS_PITCH) * sizeof(float);
  }
};

template <int BM, int BN, int TM, int TN, int CK>
__global__ void __launch_bounds__(ConvCfg<BM, BN, TM, TN, CK>::THREADS)
conv1d_simt_kernel(const float *__restrict__ x, const float *__restrict__ w,
                   const float *__restrict__ bias, float *y, int Cin, int T, int Cout, int K,
                   int dil, int pad, int y_len, int y_pitch, Epi ep) {
  using Cfg = ConvCfg<BM, BN, TM, TN, CK>;
  extern __shared__ __align__(16) float smem[];
  const int W = BN + (K - 1) * dil;
  float *xs = smem;                 // [CK][W]
  float *ws = smem + Cfg::xs_floats(W);  // [CK][K][WS_PITCH]

  const int tid = threadIdx.x;
  const int tx = tid % Cfg::NTX;
  const int ty = tid / Cfg::NTX;
  const int t0 = blockIdx.x * BN;
  const int m0 = blockIdx.y * BM;
  const int b = blockIdx.z;
  const float *xb = x + (size_t)b * Cin * T;

  float acc[TM][TN];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int q = 0; q < TN; ++q) acc[i][q] = 0.0f;

  for (int i0 = 0; i0 < Cin; i0 += CK) {
    // stage the input rows (zero outside [0, T) and beyond Cin) through
    // cp.async, all of a thread's copies in flight at once
    for (int idx = tid; idx < CK * W; idx += Cfg::THREADS) {
      const int ci = idx / W, n = idx - ci * W;
      const int tin = t0 - pad + n;
      const bool ok = i0 + ci < Cin && tin >= 0 && tin < T;
      cp_async4_zfill(xs + idx, ok ? xb + (size_t)(i0 + ci) * T + tin : xb, ok);
    }
    // stage the weights as [ci][j][m]; global order (m, ci, j) is contiguous in (ci, j)
    const int KC = CK * K;
    for (int idx = tid; idx < BM * KC; idx += Cfg::THREADS) {
      const int m = idx / KC, r = idx - m * KC;
      const int ci = r / K, j = r - ci * K;
      const bool ok = m0 + m < Cout && i0 + ci < Cin;
      cp_async4_zfill(ws + (ci * K + j) * Cfg::WS_PITCH + m,
                      ok ? w + ((size_t)(m0 + m) * Cin + i0 + ci) * K + j : w, ok);
    }
    cp_async_wait_all();
    __syncthreads();

    for (int ci = 0; ci < CK; ++ci) {
      const float *xrow = xs + ci * W + tx;
      const float *wrow = ws + (size_t)ci * K * Cfg::WS_PITCH + ty * TM;
      for (int j = 0; j < K; ++j) {
        float av[TM];
#pragma unroll
        for (int i = 0; i < TM; i += 4) {
          if constexpr (TM % 4 == 0) {
            const float4 t4 = *reinterpret_cast<const float4 *>(wrow + j * Cfg::WS_PITCH + i);
            av[i] = t4.x; av[i + 1] = t4.y; av[i + 2] = t4.z; av[i + 3] = t4.w;
          }
        }
        if constexpr (TM % 4 != 0) {
#pragma unroll
          for (int i = 0; i < TM; ++i) av[i] = wrow[j * Cfg::WS_PITCH + i];
        }
        float bv[TN];
        const float *xp = xrow + j * dil;
#pragma unroll
        for (int q = 0; q < TN; ++q) bv[q] = xp[q * Cfg::NTX];
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
          for (int q = 0; q < TN; ++q) acc[i][q] = fmaf(av[i], bv[q], acc[i][q]);
      }
    }
    __syncthreads();
  }

  // fused epilogue: all reads (bias, residual, accumulated y) first, then
  // the writes, so the loads overlap
  // (read-only path: each index is read once, by the thread that writes it;
  // the biases are read before any write too)
  float bos[TM];
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int o = m0 + ty * TM + i;
    bos[i] = (bias && o < Cout) ? __ldg(bias + o) : 0.0f;
  }
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int o = m0 + ty * TM + i;
    if (o >= Cout) continue;
    const float bo = bos[i];
    const size_t rowoff = ((size_t)b * Cout + o) * y_pitch;
#pragma unroll
    for (int q = 0; q < TN; ++q) {
      const int t = t0 + tx + q * Cfg::NTX;
      if (t < y_len) {
        float v = acc[i][q] + bo;
        if (ep.residual) v += __ldg(ep.residual + rowoff + t);
        v *= ep.scale;
        if (ep.accumulate) v += __ldg(y + rowoff + t);
        acc[i][q] = v;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int o = m0 + ty * TM + i;
    if (o >= Cout) continue;
    float *yrow = y + ((size_t)b * Cout + o) * y_pitch;
#pragma unroll
    for (int q = 0; q < TN; ++q) {
      const int t = t0 + tx + q * Cfg::NTX;
      if (t < y_len) yrow[t] = epi_final(acc[i][q], ep);
    }
  }
}

template <int BM, int BN, int TM, int TN, int CK>
bv_status run_conv(const float *x, int B, int Cin, int T, const float *w, const float *bias,
                   int Cout, int K, int dil, int pad, const Epi &ep, float *y, int y_len,
                   int y_pitch, cudaStream_t st) {
  using Cfg = ConvCfg<BM, BN, TM, TN, CK>;
  const size_t smem = Cfg::smem_bytes(K, dil);
  if (smem > 227 * 1024) return fail(BV_ERR_UNSUPPORTED, "conv1d: K*dilation too large");
  auto kern = conv1d_simt_kernel<BM, BN, TM, TN, CK>;
  BV_TRY(ensure_dynamic_smem((const void *)kern, smem, "conv1d smem attribute"));
  dim3 grid((y_len + BN - 1) / BN, (Cout + BM - 1) / BM, B);
  if (grid.y > 65535 || grid.z > 65535) return fail(BV_ERR_SHAPE, "conv1d: grid too large");
  {
    const double outs = (double)B * Cout * y_len;
    LaunchTimer tm(st, "conv1d_simt", 2.0 * outs * Cin * K,
                   4.0 * ((double)B * Cin * T + (double)Cout * Cin * K +
                          outs * (1 + (ep.residual ? 1 : 0) + ep.accumulate)));
    kern<<<grid, Cfg::THREADS, smem, st>>>(x, w, bias, y, Cin, T, Cout, K, dil, pad, y_len,
                                            y_pitch, ep);
  }
  count_launch();
  return check_launch("conv1d_simt_kernel");
}

}  // namespace

bv_status launch_conv1d(const float *x, int B, int Cin, int T, const float *w, const float *bias,
                        int Cout, int K, int dil, int pad, const Epi &ep, float *y, int y_len,
                        int y_pitch, cudaStream_t st, const float *w_split) {
  if (B <= 0 || y_len <= 0) return BV_OK;
  if (conv1d_tc_supported(Cin, Cout, K, dil) && (reinterpret_cast<uintptr_t>(w) & 15u) == 0 &&
      (reinterpret_cast<uintptr_t>(w_split) & 15u) == 0)
    return launch_conv1d_tc(x, B, Cin, T, w, w_split, bias, Cout, K, dil, pad, ep, y, y_len, y_pitch,
                            st);
  if (conv1d_small_supported(Cin, Cout, K, dil))
    return launch_conv1d_small(x, B, Cin, T, w, bias, Cout, K, dil, pad, ep, y, y_len, y_pitch,
                               st);
  if (Cout >= 96)
    return run_conv<128, 128, 8, 8, 8>(x, B, Cin, T, w, bias, Cout, K, dil, pad, ep, y, y_len,
                                       y_pitch, st);
  if (Cout >= 24)
    return run_conv<32, 256, 4, 8, 8>(x, B, Cin, T, w, bias, Cout, K, dil, pad, ep, y, y_len,
                                      y_pitch, st);
  if (Cout > 4)
    return run_conv<16, 256, 2, 8, 8>(x, B, Cin, T, w, bias, Cout, K, dil, pad, ep, y, y_len,
                                      y_pitch, st);
  return run_conv<4, 512, 1, 8, 8>(x, B, Cin, T, w, bias, Cout, K, dil, pad, ep, y, y_len,
                                   y_pitch, st);
}

}  // namespace bv
