// The latent front end of the MiniMax-H3 audio VAE decode (docs.rs
// cortiq-engine 0.5.74 audiovae.rs, `AudioVae::decode` and `from_cmf`): the
// normalised latents arrive as z [C, S, T] (channel ci of side s at
// (ci S + s) T + t; stereo is S = 2), are de-normalised per channel,
//   lat[s, ci, t] = z[ci, s, t] std[ci] + mean[ci],
// and projected by `dec_in_proj`, a one-tap Conv1d,
//   out[s, o, t] = bias[o] + sum_ci w[o, ci] lat[s, ci, t],
// giving the decoder's input [S, Cout, T].  One thread per (s, t), output
// channels in groups of 8 (the latent column is re-read from L1 per group);
// reads and writes are coalesced along t.
#include "common.cuh"

namespace bv {
namespace {

constexpr int FE_GROUP = 8;

__global__ void __launch_bounds__(256)
latent_front_end_kernel(const float *__restrict__ z, int C, int S, int T,
                        const float *__restrict__ mean, const float *__restrict__ stdv,
                        const float *__restrict__ w, const float *__restrict__ bias, int Cout,
                        float *__restrict__ out) {
  const long long n = (long long)S * T;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int s = (int)(i / T), t = (int)(i - (long long)s * T);
    for (int o0 = 0; o0 < Cout; o0 += FE_GROUP) {
      float acc[FE_GROUP];
#pragma unroll
      for (int q = 0; q < FE_GROUP; ++q)
        acc[q] = (bias && o0 + q < Cout) ? __ldg(bias + o0 + q) : 0.0f;
      for (int ci = 0; ci < C; ++ci) {
        const float lat =
            fmaf(__ldg(z + ((size_t)ci * S + s) * T + t), __ldg(stdv + ci), __ldg(mean + ci));
#pragma unroll
        for (int q = 0; q < FE_GROUP; ++q)
          if (o0 + q < Cout) acc[q] = fmaf(__ldg(w + (size_t)(o0 + q) * C + ci), lat, acc[q]);
      }
#pragma unroll
      for (int q = 0; q < FE_GROUP; ++q)
        if (o0 + q < Cout) out[((size_t)s * Cout + o0 + q) * T + t] = acc[q];
    }
  }
}

}  // namespace

bv_status launch_latent_front_end(const float *z, int C, int S, int T, const float *mean,
                                  const float *stdv, const float *w, const float *bias, int Cout,
                                  float *out, cudaStream_t st) {
  const long long n = (long long)S * T;
  if (n <= 0) return BV_OK;
  const long long blocks = (n + 255) / 256;
  {
    LaunchTimer tm(st, "front_end", 2.0 * n * C * Cout,
                   4.0 * (double)n * (C + Cout) + 4.0 * (double)Cout * C);
    latent_front_end_kernel<<<(unsigned)(blocks < 148 * 16 ? blocks : 148 * 16), 256, 0, st>>>(
        z, C, S, T, mean, stdv, w, bias, Cout, out);
  }
  count_launch();
  return check_launch("latent_front_end_kernel");
}

}  // namespace bv
