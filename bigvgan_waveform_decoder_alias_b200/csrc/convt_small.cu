// ConvTranspose1d for narrow layers (at most 64 input and 32 output
// channels) on the FP32 pipe, as a polyphase gather with bias:
//
//   y[o, p] = bias[o] + sum_i sum_{m < NT} x[i, P - m] w[i, o, r + S m],
//   p = S P + r - pad, r < S, NT = ceil(K / S),
// terms with r + S m >= K or P - m outside [0, T) left out (the pages'
// scatter `out[o, t S + j - pad] += x[i, t] w[i, o, j]`, docs.rs
// cortiq-engine audiovae.rs `ConvT1d::apply`, ltxaudio.rs
// `ConvT1d::forward`, gathered per output phase).
//
// A CTA takes CT_P consecutive input positions P of one batch row, every
// output phase and every output channel: S groups of 128 threads, group r
// computing phase r (warp-uniform, so weight reads are broadcasts), each
// thread 4 consecutive P x COUT channels in registers.  The input rows
// (zero outside [0, T)) are staged in chunks of CT_CI channels with
// zero-filling cp.async; all the weights are staged once, reordered to
// [i][j][o] so that the output channels of one (input channel, tap) are a
// run of 16-byte broadcast reads.
#include "common.cuh"

namespace bv {
namespace {

constexpr int CT_P = 512;       // input positions per CTA
constexpr int CT_PER = 4;       // consecutive positions per thread
constexpr int CT_GROUP = CT_P / CT_PER;  // threads per phase
constexpr int CT_CI = 16;       // input channels per staged chunk
constexpr int CT_MAX_NT = 4;    // taps per phase
constexpr int CT_MAX_CIN = 64;
constexpr int CT_MAX_COUT = 32;

template <int COUT>
__global__ void __launch_bounds__(256)
convt_small_kernel(const float *__restrict__ x, const float *__restrict__ w,
                   const float *__restrict__ bias, float *__restrict__ y, int Cin, int T,
                   int Cout, int K, int S, int NT, int pad, int Tout) {
  extern __shared__ __align__(16) float sm[];
  const int XW = (CT_P + NT - 1 + 3) & ~3;        // staged row width
  float *ws = sm;                                  // [Cin][S NT][COUT]
  float *xs = sm + Cin * S * NT * COUT;            // [CT_CI][XW]
  __shared__ float bias_s[COUT];
  const int P0 = blockIdx.x * CT_P, b = blockIdx.y;
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int r = tid / CT_GROUP, q = tid - r * CT_GROUP;  // phase, thread in the group

  for (int idx = tid; idx < Cin * S * NT * COUT; idx += nthr) {
    const int o = idx % COUT, ij = idx / COUT;
    const int i = ij / (S * NT), j = ij - i * (S * NT);
    const bool ok = o < Cout && j < K;
    cp_async4_zfill(ws + idx, ok ? w + ((size_t)i * Cout + o) * K + j : w, ok);
  }
  if (tid < COUT) bias_s[tid] = (bias && tid < Cout) ? __ldg(bias + tid) : 0.0f;

  float acc[COUT][CT_PER];
#pragma unroll
  for (int o = 0; o < COUT; ++o)
#pragma unroll
    for (int e = 0; e < CT_PER; ++e) acc[o][e] = 0.0f;
  const float *xb = x + (size_t)b * Cin * T;
  const int pl = CT_PER * q;  // this thread's positions P0 + pl .. + 3
  for (int i0 = 0; i0 < Cin; i0 += CT_CI) {
    const int ni = Cin - i0 < CT_CI ? Cin - i0 : CT_CI;
    __syncthreads();  // the previous chunk has been read
    // staged column n holds x[P0 - (NT - 1) + n]
    for (int idx = tid; idx < ni * XW; idx += nthr) {
      const int ii = idx / XW, n = idx - ii * XW;
      const int t = P0 - (NT - 1) + n;
      const bool ok = t >= 0 && t < T && n < CT_P + NT - 1;
      cp_async4_zfill(xs + idx, ok ? xb + (size_t)(i0 + ii) * T + t : xb, ok);
    }
    cp_async_wait_all();
    __syncthreads();
    if (r < S) {
      for (int ii = 0; ii < ni; ++ii) {
        const float *xr = xs + ii * XW + pl + (NT - 1);  // x[P0 + pl + e - m] at xr[e - m]
        const float4 *wr = reinterpret_cast<const float4 *>(ws + (size_t)(i0 + ii) * S * NT * COUT);
#pragma unroll
        for (int m = 0; m < CT_MAX_NT; ++m) {
          if (m < NT) {
            float xv[CT_PER];
#pragma unroll
            for (int e = 0; e < CT_PER; ++e) xv[e] = xr[e - m];
            const float4 *wj = wr + (r + S * m) * (COUT / 4);
#pragma unroll
            for (int o4 = 0; o4 < COUT / 4; ++o4) {
              const float4 wv = wj[o4];
#pragma unroll
              for (int e = 0; e < CT_PER; ++e) {
                acc[4 * o4][e] = fmaf(wv.x, xv[e], acc[4 * o4][e]);
                acc[4 * o4 + 1][e] = fmaf(wv.y, xv[e], acc[4 * o4 + 1][e]);
                acc[4 * o4 + 2][e] = fmaf(wv.z, xv[e], acc[4 * o4 + 2][e]);
                acc[4 * o4 + 3][e] = fmaf(wv.w, xv[e], acc[4 * o4 + 3][e]);
              }
            }
          }
        }
      }
    }
  }
  if (r >= S) return;
  float *yb = y + (size_t)b * Cout * Tout;
#pragma unroll
  for (int o = 0; o < COUT; ++o) {
    if (o >= Cout) break;
    const float bo = bias_s[o];
#pragma unroll
    for (int e = 0; e < CT_PER; ++e) {
      const long long p = (long long)S * (P0 + pl + e) + r - pad;
      if (p >= 0 && p < Tout) yb[(size_t)o * Tout + p] = acc[o][e] + bo;
    }
  }
}

}  // namespace

// One 128-thread group per phase within the 256-thread launch bound: strides
// 1 and 2 (the decoders' narrow stages are stride 2).
bool conv_transpose1d_small_supported(int Cin, int Cout, int K, int S) {
  const int nt = (K + S - 1) / S;
  return Cin >= 1 && Cin <= CT_MAX_CIN && Cout >= 1 && Cout <= CT_MAX_COUT && S >= 1 &&
         S * CT_GROUP <= 256 && nt >= 1 && nt <= CT_MAX_NT;
}

bv_status launch_conv_transpose1d_small(const float *x, int B, int Cin, int T, const float *w,
                                        const float *bias, int Cout, int K, int S, int pad,
                                        float *y, cudaStream_t st) {
  const int Tout = (T - 1) * S + K - 2 * pad;
  if (B <= 0 || Tout <= 0) return BV_OK;
  const int NT = (K + S - 1) / S;
  const int threads = S * CT_GROUP;
  const int XW = (CT_P + NT - 1 + 3) & ~3;
  const int cout4 = (Cout + 3) / 4 * 4;
  const int COUT = cout4 <= 8 ? 8 : cout4 <= 12 ? 12 : cout4 <= 16 ? 16 : cout4 <= 24 ? 24 : 32;
  const size_t smem = ((size_t)Cin * S * NT * COUT + (size_t)CT_CI * XW) * sizeof(float);
  // input positions P of the outputs: [0, T + NT - 1) (the last outputs of a
  // row gather positions past the input's end, where only earlier taps hit)
  dim3 grid((T + NT - 1 + CT_P - 1) / CT_P, B);
  if (grid.y > 65535) return fail(BV_ERR_SHAPE, "convt_small: grid");
  LaunchTimer tm(st, "conv_transpose1d", 2.0 * B * Cin * (double)Cout * K * T,
                 4.0 * ((double)B * Cin * T + (double)Cin * Cout * K + (double)B * Cout * Tout));
#define BV_CT_CASE(N)                                                                        \
  case N: {                                                                                  \
    BV_TRY(ensure_dynamic_smem((const void *)convt_small_kernel<N>, smem, "convt_small smem")); \
    convt_small_kernel<N><<<grid, threads, smem, st>>>(x, w, bias, y, Cin, T, Cout, K, S, NT,  \
                                                       pad, Tout);                           \
    break;                                                                                   \
  }
  switch (COUT) {
    BV_CT_CASE(8)
    BV_CT_CASE(12)
    BV_CT_CASE(16)
    BV_CT_CASE(24)
    BV_CT_CASE(32)
    default:
      return fail(BV_ERR_UNSUPPORTED, "convt_small: Cout %d", Cout);
  }
#undef BV_CT_CASE
  count_launch();
  return check_launch("convt_small_kernel");
}

}  // namespace bv
