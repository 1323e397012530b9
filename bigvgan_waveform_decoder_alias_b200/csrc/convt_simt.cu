// ConvTranspose1d as a polyphase gather on the FP32 pipe (no scatter, no
// atomics), bias fused.
//
// The pages' scatter (docs.rs cortiq-engine audiovae.rs `ConvT1d::apply`,
// ltxaudio.rs `ConvT1d::forward`):  y[o, t s + j - pad] += x[i, t] w[i, o, j].
// Gathered per output p: with r = (p + pad) mod s and P = (p + pad) div s,
//   y[o, p] = bias[o] + sum_i sum_{m: j = r + s m < K} x[i, P - m] w[i, o, j].
// Every output of one phase r uses the same taps, so a thread whose outputs
// are all p = p0 + tx + NTX k with NTX a multiple of s keeps one phase: its
// weights are shared by all its outputs (an outer product, as in a GEMM),
// and consecutive threads still write consecutive samples.
#include "common.cuh"

namespace bv {
namespace {

constexpr int CK = 8;  // input channels per staged chunk

__host__ __device__ constexpr int gcd_i(int a, int b) { return b == 0 ? a : gcd_i(b, a % b); }

template <int TM, int TP>
__global__ void __launch_bounds__(256)
convt_simt_kernel(const float *__restrict__ x, const float *__restrict__ w,
                  const float *__restrict__ bias, float *__restrict__ y, int Cin, int T, int Cout,
                  int K, int S, int pad, int Tout, int NTX, int NTAP) {
  extern __shared__ __align__(16) float smem[];
  const int NTY = blockDim.x / NTX;
  const int BM = NTY * TM;
  const int BP = NTX * TP;
  const int WSP = BM + 4;                      // weight row pitch in smem
  const int p0 = blockIdx.x * BP;              // multiple of S (BP is)
  const int m0 = blockIdx.y * BM;
  const int b = blockIdx.z;
  const int P_lo = (p0 + pad) / S - (NTAP - 1);
  const int P_hi = (p0 + BP - 1 + pad) / S;
  const int WX = P_hi - P_lo + 1;
  float *xs = smem;                            // [CK][WX]
  float *ws = smem + ((CK * WX + 3) & ~3);     // [CK][K][WSP], 16-byte aligned

  const int tid = threadIdx.x;
  const int tx = tid % NTX, ty = tid / NTX;
  const int r = (tx + pad) % S;                // this thread's phase (p0 % S == 0)
  const int Pt = (p0 + tx + pad) / S - P_lo;   // staged index of P for k = 0
  const int dP = NTX / S;                      // P step between a thread's outputs
  const float *xb = x + (size_t)b * Cin * T;

  float acc[TM][TP];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int k = 0; k < TP; ++k) acc[i][k] = 0.0f;

  for (int i0 = 0; i0 < Cin; i0 += CK) {
    // staged through cp.async (zero-filled outside the input and the channels)
    for (int idx = tid; idx < CK * WX; idx += blockDim.x) {
      const int ci = idx / WX, q = idx - ci * WX;
      const int tin = P_lo + q;
      const bool ok = i0 + ci < Cin && tin >= 0 && tin < T;
      cp_async4_zfill(xs + idx, ok ? xb + (size_t)(i0 + ci) * T + tin : xb, ok);
    }
    // w[i, o, j]: contiguous over (o, j) for a fixed i
    const int MK = BM * K;
    for (int idx = tid; idx < CK * MK; idx += blockDim.x) {
      const int ci = idx / MK, rem = idx - ci * MK;
      const int m = rem / K, j = rem - m * K;
      const bool ok = i0 + ci < Cin && m0 + m < Cout;
      cp_async4_zfill(ws + (ci * K + j) * WSP + m,
                      ok ? w + ((size_t)(i0 + ci) * Cout + m0 + m) * K + j : w, ok);
    }
    cp_async_wait_all();
    __syncthreads();
    for (int ci = 0; ci < CK; ++ci) {
      for (int mm = 0; mm < NTAP; ++mm) {
        const int j = r + S * mm;
        if (j >= K) break;
        const float *wp = ws + (ci * K + j) * WSP + ty * TM;
        float av[TM];
#pragma unroll
        for (int i = 0; i < TM; i += 4) {
          const float4 t4 = *reinterpret_cast<const float4 *>(wp + i);
          av[i] = t4.x; av[i + 1] = t4.y; av[i + 2] = t4.z; av[i + 3] = t4.w;
        }
        const float *xp = xs + ci * WX + Pt - mm;
        float bv[TP];
#pragma unroll
        for (int k = 0; k < TP; ++k) bv[k] = xp[k * dP];
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
          for (int k = 0; k < TP; ++k) acc[i][k] = fmaf(av[i], bv[k], acc[i][k]);
      }
    }
    __syncthreads();
  }

  // the biases are read before any output is written (a load between the
  // stores would wait a full round trip each)
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
    float *yrow = y + ((size_t)b * Cout + o) * Tout;
#pragma unroll
    for (int k = 0; k < TP; ++k) {
      const int p = p0 + tx + k * NTX;
      if (p < Tout) yrow[p] = acc[i][k] + bo;
    }
  }
}

}  // namespace

bv_status launch_conv_transpose1d(const float *x, int B, int Cin, int T, const float *w,
                                  const float *bias, int Cout, int K, int S, int pad, float *y,
                                  cudaStream_t st) {
  const int Tout = (T - 1) * S + K - 2 * pad;
  if (B <= 0 || Tout <= 0) return BV_OK;
  if (conv_transpose1d_small_supported(Cin, Cout, K, S))
    return launch_conv_transpose1d_small(x, B, Cin, T, w, bias, Cout, K, S, pad, y, st);
  const int NTX = S / gcd_i(S, 32) * 32;  // lcm(S, 32): a multiple of both
  if (NTX > 256) return fail(BV_ERR_UNSUPPORTED, "conv_transpose1d: stride %d", S);
  const int NTY = 256 / NTX;
  const int threads = NTX * NTY;
  const int NTAP = (K + S - 1) / S;
  const bool wide = NTY <= 2;  // few thread rows: give each thread more channels
  const int TM = wide ? 16 : 8, TP = 4;
  const int BM = NTY * TM, BP = NTX * TP;
  const int WX = BP / S + NTAP + 1;
  const size_t smem = ((size_t)((CK * WX + 3) & ~3) + (size_t)CK * K * (BM + 4)) * sizeof(float);
  if (smem > 200 * 1024) return fail(BV_ERR_UNSUPPORTED, "conv_transpose1d: kernel too long");
  dim3 grid((Tout + BP - 1) / BP, (Cout + BM - 1) / BM, B);
  if (grid.y > 65535 || grid.z > 65535) return fail(BV_ERR_SHAPE, "conv_transpose1d: grid");
  LaunchTimer tm(st, "conv_transpose1d", 2.0 * B * Cin * (double)Cout * K * T,
                 4.0 * ((double)B * Cin * T + (double)Cin * Cout * K + (double)B * Cout * Tout));
  if (wide) {
    auto kern = convt_simt_kernel<16, 4>;
    BV_TRY(ensure_dynamic_smem((const void *)kern, smem, "convt smem attribute"));
    kern<<<grid, threads, smem, st>>>(x, w, bias, y, Cin, T, Cout, K, S, pad, Tout, NTX, NTAP);
  } else {
    auto kern = convt_simt_kernel<8, 4>;
    BV_TRY(ensure_dynamic_smem((const void *)kern, smem, "convt smem attribute"));
    kern<<<grid, threads, smem, st>>>(x, w, bias, y, Cin, T, Cout, K, S, pad, Tout, NTX, NTAP);
  }
  count_launch();
  return check_launch("convt_simt_kernel");
}

}  // namespace bv
