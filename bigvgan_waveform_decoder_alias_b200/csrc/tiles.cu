// Time tiling of a long latent: gather the tiles into a batch, and stitch the
// decoded tiles back, averaging samples over the tiles that cover them (the
// overlapping-window rule of docs.rs cortiq-engine music3.rs
// `Music3Dit::forward_windowed`).
#include "common.cuh"
#include "tiles.cuh"

namespace bv {
namespace {

// zt[j, c, f] = z[b, c, k step + f] for unit u = u0 + j = k B + b (tile k of
// side b), j < n_units, tiles of length len.
__global__ void gather_tiles_kernel(const float *__restrict__ z, float *__restrict__ zt, int B,
                                    int C, int frames, int step, int len, long long u0,
                                    long long n_units) {
  const long long total = n_units * C * len;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int f = (int)(i % len);
    long long r = i / len;
    const int c = (int)(r % C);
    const long long u = u0 + r / C;
    const int b = (int)(u % B);
    const long long k = u / B;
    zt[i] = z[((long long)b * C + c) * frames + k * step + f];
  }
}

// y[b, o, t]: mean over the tiles covering sample t.  Tile k covers samples
// [k step hop, k step hop + len_k hop); group g holds tiles [k0_g, k0_g + n_g)
// of length len_g, decoded as rows (k - k0_g) * B + b.
__global__ void stitch_tiles_kernel(TileGroups g, float *__restrict__ y, int B, int O,
                                    long long L, int step_samples) {
  const long long total = (long long)B * O * L;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long t = i % L;
    const long long bo = i / L;
    const int o = (int)(bo % O), b = (int)(bo / O);
    // tiles k with k * step <= t < k * step + len_k: k in [ (t - maxlen) / step, t / step ]
    float sum = 0.0f;
    int cnt = 0;
    const long long khi = t / step_samples;
    for (long long k = khi; k >= 0; --k) {
      const long long start = k * step_samples;
      int gi = -1;
      for (int q = 0; q < g.n; ++q)
        if (k >= g.k0[q] && k < g.k0[q] + g.count[q]) gi = q;
      if (gi < 0) continue;
      const long long len = g.len_samples[gi];
      if (t - start >= len) {
        if (t - start >= g.max_len_samples) break;
        continue;
      }
      const long long row = (k - g.k0[gi]) * B + b;
      sum += g.data[gi][(row * O + o) * g.pitch[gi] + (t - start)];
      ++cnt;
    }
    y[i] = cnt ? sum / (float)cnt : 0.0f;
  }
}

// acc[i] = ((acc[i] + p[0][i]) + p[1][i]) + ... in that order
__global__ void add_parts_kernel(float *__restrict__ acc, Parts parts, long long n) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += stride) {
    float v = acc[i];
    for (int q = 0; q < parts.n; ++q) v += __ldg(parts.p[q] + i);
    acc[i] = v;
  }
}

}  // namespace

bv_status launch_add_parts(float *acc, const Parts &parts, long long n, cudaStream_t st) {
  if (n <= 0 || parts.n <= 0) return BV_OK;
  const int threads = 256;
  const long long blocks = (n + threads - 1) / threads;
  {
    LaunchTimer tm(st, "stage_sum", 0.0, 4.0 * (double)n * (parts.n + 2));
    add_parts_kernel<<<(unsigned)(blocks < 148 * 16 ? blocks : 148 * 16), threads, 0, st>>>(
        acc, parts, n);
  }
  count_launch();
  return check_launch("add_parts_kernel");
}

bv_status launch_gather_tiles(const float *z, float *zt, int B, int C, int frames, int step,
                              int len, long long u0, long long n_units, cudaStream_t st) {
  const long long total = n_units * C * len;
  if (total <= 0) return BV_OK;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  LaunchTimer tm(st, "tiles", 0.0, 8.0 * (double)total);
  gather_tiles_kernel<<<(unsigned)(blocks < 148 * 32 ? blocks : 148 * 32), threads, 0, st>>>(
      z, zt, B, C, frames, step, len, u0, n_units);
  count_launch();
  return check_launch("gather_tiles_kernel");
}

bv_status launch_stitch_tiles(const TileGroups &g, float *y, int B, int O, long long L,
                              int step_samples, cudaStream_t st) {
  const long long total = (long long)B * O * L;
  if (total <= 0) return BV_OK;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  LaunchTimer tm(st, "tiles", 0.0, 8.0 * (double)total);
  stitch_tiles_kernel<<<(unsigned)(blocks < 148 * 32 ? blocks : 148 * 32), threads, 0, st>>>(
      g, y, B, O, L, step_samples);
  count_launch();
  return check_launch("stitch_tiles_kernel");
}

}  // namespace bv
