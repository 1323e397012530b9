// The latent front end of the MiniMax-H3 audio VAE decode (docs.rs
// cortiq-engine 0.5.74 audiovae.rs, `AudioVae::decode` and `from_cmf`): the
// normalised latents arrive as z [C, S, T] (channel ci of side s at
// (ci S + s) T + t; stereo is S = 2), are de-normalised per channel,
//   lat[s, ci, t] = z[ci, s, t] std[ci] + mean[ci],
// and projected by `dec_in_proj`, a one-tap Conv1d,
//   out[s, o, t] = bias[o] + sum_ci w[o, ci] lat[s, ci, t],
// giving the decoder's input [S, Cout, T].  A CTA takes 256 consecutive
// (s, t) positions and 8 output channels (grid y): it stages the 8 weight
// rows and the de-normalisation constants in shared memory, then each thread
// reads its latent column once (coalesced along t) into 8 accumulators.
#include "common.cuh"

namespace bv {
namespace {

constexpr int FE_GROUP = 8;
constexpr int FE_THREADS = 256;

__global__ void __launch_bounds__(FE_THREADS)
latent_front_end_kernel(const float *__restrict__ z, int C, int S, int T,
                        const float *__restrict__ mean, const float *__restrict__ stdv,
                        const float *__restrict__ w, const float *__restrict__ bias, int Cout,
                        float *__restrict__ out) {
  extern __shared__ __align__(16) float fe_sm[];
  float *ws = fe_sm;                 // [C][FE_GROUP] weights of this CTA's channels
  float *ms = fe_sm + FE_GROUP * C;  // [C] (std, mean) pairs
  const int o0 = blockIdx.y * FE_GROUP;
  for (int i = threadIdx.x; i < FE_GROUP * C; i += FE_THREADS) {
    const int ci = i / FE_GROUP, q = i - ci * FE_GROUP;
    ws[i] = o0 + q < Cout ? __ldg(w + (size_t)(o0 + q) * C + ci) : 0.0f;
  }
  for (int ci = threadIdx.x; ci < C; ci += FE_THREADS) {
    ms[2 * ci] = __ldg(stdv + ci);
    ms[2 * ci + 1] = __ldg(mean + ci);
  }
  __syncthreads();
  const long long n = (long long)S * T;
  const long long i = blockIdx.x * (long long)FE_THREADS + threadIdx.x;
  if (i >= n) return;
  const int s = (int)(i / T), t = (int)(i - (long long)s * T);
  float acc[FE_GROUP];
#pragma unroll
  for (int q = 0; q < FE_GROUP; ++q) acc[q] = (bias && o0 + q < Cout) ? __ldg(bias + o0 + q) : 0.0f;
  const float *zc = z + (size_t)s * T + t;  // channel ci at zc + ci S T
  const size_t cstride = (size_t)S * T;
  for (int ci = 0; ci < C; ++ci) {
    const float lat = fmaf(__ldg(zc + ci * cstride), ms[2 * ci], ms[2 * ci + 1]);
    const float4 w0 = *reinterpret_cast<const float4 *>(ws + FE_GROUP * ci);
    const float4 w1 = *reinterpret_cast<const float4 *>(ws + FE_GROUP * ci + 4);
    acc[0] = fmaf(w0.x, lat, acc[0]);
    acc[1] = fmaf(w0.y, lat, acc[1]);
    acc[2] = fmaf(w0.z, lat, acc[2]);
    acc[3] = fmaf(w0.w, lat, acc[3]);
    acc[4] = fmaf(w1.x, lat, acc[4]);
    acc[5] = fmaf(w1.y, lat, acc[5]);
    acc[6] = fmaf(w1.z, lat, acc[6]);
    acc[7] = fmaf(w1.w, lat, acc[7]);
  }
#pragma unroll
  for (int q = 0; q < FE_GROUP; ++q)
    if (o0 + q < Cout) out[((size_t)s * Cout + o0 + q) * T + t] = acc[q];
}

}  // namespace

bv_status launch_latent_front_end(const float *z, int C, int S, int T, const float *mean,
                                  const float *stdv, const float *w, const float *bias, int Cout,
                                  float *out, cudaStream_t st) {
  const long long n = (long long)S * T;
  if (n <= 0 || Cout <= 0) return BV_OK;
  const size_t smem = (size_t)(FE_GROUP + 2) * C * sizeof(float);
  if (smem > 200 * 1024) return fail(BV_ERR_UNSUPPORTED, "front end: %d latent channels", C);
  const long long bx = (n + FE_THREADS - 1) / FE_THREADS;
  const int by = (Cout + FE_GROUP - 1) / FE_GROUP;
  if (bx > 0x7fffffffLL || by > 65535) return fail(BV_ERR_SHAPE, "front end: grid");
  BV_TRY(ensure_dynamic_smem((const void *)latent_front_end_kernel, smem, "front end smem"));
  {
    LaunchTimer tm(st, "front_end", 2.0 * n * C * Cout,
                   4.0 * (double)n * (C + Cout) + 4.0 * (double)Cout * C);
    latent_front_end_kernel<<<dim3((unsigned)bx, (unsigned)by), FE_THREADS, smem, st>>>(
        z, C, S, T, mean, stdv, w, bias, Cout, out);
  }
  count_launch();
  return check_launch("latent_front_end_kernel");
}

}  // namespace bv
