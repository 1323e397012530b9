// Fused alias-free activation: 2x kaiser-sinc upsample -> SnakeBeta -> 2x
// lowpass downsample, one pass over HBM (read x, write y).  The 2x signal
// lives only in shared memory.
//
// Definition (per row of length n, 12-tap filters f_up, f_down), from
// docs.rs cortiq-engine audiovae.rs `Activation1d::apply` / `fir_pad` and
// ltxaudio.rs `Aliasing::{upsample, downsample}`:
//   u[2p]   = 2 sum_{l<6} f_up[2l+1] x[clamp(p + 2 - l)]
//   u[2p+1] = 2 sum_{l<6} f_up[2l]   x[clamp(p + 3 - l)]
//   v[m]    = u[m] + sin^2(a u[m]) inv_b,  a = e^{log_alpha}, inv_b = 1/(e^{log_beta} + eps)
//   y[t]    = sum_{j<12} f_down[j] v[clamp(2t + j - 5, 0, 2n-1)]
// (the polyphase form of the pages' replicate pad 5 / stride-2 transposed
// FIR / trim 15 / replicate pad 5|6 / stride-2 FIR).
//
// Persistent CTAs walk row tiles of TILE outputs.  While a CTA computes one
// tile, the next tile's input x[t0-8 .. t0+TILE+8) (clamped at the row ends)
// is already streaming into the other half of a double buffer with cp.async
// (16-byte copies when the row is 16-byte aligned and the tile is interior).
// Per tile: stage A computes v[2 t0 - 6 + k], k < 2 TILE + 12, into shared
// memory; stage B filters v into the TILE outputs.
#include "common.cuh"
#include "sin2.cuh"

namespace bv {
namespace {

constexpr int TILE = 1024;         // outputs per tile
constexpr int THREADS = 256;       // 4 outputs and 8 up-sampled values each
constexpr int XS = TILE + 16;      // x[t0 - 8 + i]
constexpr int VS = 2 * TILE + 16;  // v[2 t0 - 6 + k], k < 2 TILE + 12 used

struct Taps {
  float up2[12];  // 2 * f_up
  float dn[12];
};

__device__ __forceinline__ float snake(float u, float a, float inv_b) {
  return fmaf(sin_squared(a * u), inv_b, u);
}

// u at phase r (0: even output index, 1: odd) from 6 consecutive x values
// x0..x5 = x[p + r - 3 .. p + r + 2]:  u[2p+r] = sum_l 2 f[2l+1-r] x[p+2+r-l],
// where term l pairs with x_{5-l}.
__device__ __forceinline__ float up_phase(const Taps &tp, int r, float x0, float x1, float x2,
                                          float x3, float x4, float x5) {
  if (r == 0) {
    return tp.up2[1] * x5 + tp.up2[3] * x4 + tp.up2[5] * x3 + tp.up2[7] * x2 + tp.up2[9] * x1 +
           tp.up2[11] * x0;
  }
  return tp.up2[0] * x5 + tp.up2[2] * x4 + tp.up2[4] * x3 + tp.up2[6] * x2 + tp.up2[8] * x1 +
         tp.up2[10] * x0;
}

__device__ __forceinline__ void cp_async4(float *dst, const float *src) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16(float *dst, const float *src) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Issue the copies of tile `tile_id`'s input into xs (x[t0 - 8 + i], clamped).
__device__ __forceinline__ void issue_tile(const float *__restrict__ x, float *xs,
                                           long long tile_id, int tiles_per_row, int T, int tid) {
  const long long row = tile_id / tiles_per_row;
  const int t0 = (int)(tile_id - row * tiles_per_row) * TILE;
  const float *xr = x + row * (long long)T;
  const bool vec =
      ((reinterpret_cast<uintptr_t>(xr) & 15u) == 0) && (t0 >= 8) && (t0 + TILE + 8 <= T);
  if (vec) {
    const float *src = xr + t0 - 8;
    for (int c = tid; c < XS / 4; c += THREADS) cp_async16(xs + 4 * c, src + 4 * c);
  } else {
    for (int i = tid; i < XS; i += THREADS) {
      int p = t0 - 8 + i;
      p = p < 0 ? 0 : (p > T - 1 ? T - 1 : p);
      cp_async4(xs + i, xr + p);
    }
  }
}

__global__ void __launch_bounds__(THREADS)
activation_kernel(const float *__restrict__ x, float *__restrict__ y, int C, int T,
                  int tiles_per_row, long long n_tiles, const float *__restrict__ log_alpha,
                  const float *__restrict__ log_beta, const float *__restrict__ f_up,
                  const float *__restrict__ f_dn, float eps) {
  __shared__ __align__(16) float xs[2][XS];
  __shared__ __align__(16) float vs[VS];
  const int tid = threadIdx.x;

  Taps tp;
#pragma unroll
  for (int j = 0; j < 12; ++j) {
    tp.up2[j] = 2.0f * __ldg(f_up + j);
    tp.dn[j] = __ldg(f_dn + j);
  }

  long long tile_id = blockIdx.x;
  if (tile_id < n_tiles) issue_tile(x, xs[0], tile_id, tiles_per_row, T, tid);
  cp_async_commit();
  int buf = 0;
  for (; tile_id < n_tiles; tile_id += gridDim.x, buf ^= 1) {
    const long long next = tile_id + gridDim.x;
    if (next < n_tiles) issue_tile(x, xs[buf ^ 1], next, tiles_per_row, T, tid);
    cp_async_commit();
    cp_async_wait<1>();  // this tile's copies are done; the next tile's may be in flight
    __syncthreads();

    const long long row = tile_id / tiles_per_row;
    const int t0 = (int)(tile_id - row * tiles_per_row) * TILE;
    const int c = (int)(row % C);
    const float a = expf(__ldg(log_alpha + c));
    const float inv_b = 1.0f / (expf(__ldg(log_beta + c)) + eps);
    const float *xb = xs[buf];

    // ---- stage A: v[m] for m = 2 t0 - 6 + k, k in [0, 2 TILE + 12)
    const bool interior = (2 * t0 - 6 >= 0) && (2 * t0 + 2 * TILE + 5 <= 2 * T - 1);
    if (interior) {
      // k = 2q + r, p = t0 - 3 + q; x[p + r - 3 + k'] = x[t0 - 6 + q + r + k'] sits at
      // xb[2 + q + r + k'].  Thread owns q in [4 tid, 4 tid + 4).
      const int q0 = 4 * tid;
      const float4 w0 = *reinterpret_cast<const float4 *>(xb + q0);
      const float4 w1 = *reinterpret_cast<const float4 *>(xb + q0 + 4);
      const float4 w2 = *reinterpret_cast<const float4 *>(xb + q0 + 8);
      const float xw[12] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y,
                            w1.z, w1.w, w2.x, w2.y, w2.z, w2.w};
      float vv[8];
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int b0 = 2 + qq + r;
          const float u = up_phase(tp, r, xw[b0], xw[b0 + 1], xw[b0 + 2], xw[b0 + 3],
                                   xw[b0 + 4], xw[b0 + 5]);
          vv[2 * qq + r] = snake(u, a, inv_b);
        }
      }
      *reinterpret_cast<float4 *>(vs + 2 * q0) = make_float4(vv[0], vv[1], vv[2], vv[3]);
      *reinterpret_cast<float4 *>(vs + 2 * q0 + 4) = make_float4(vv[4], vv[5], vv[6], vv[7]);
      if (tid < 12) {  // k in [2 TILE, 2 TILE + 12): q in [TILE, TILE + 6)
        const int k = 2 * TILE + tid;
        const int q = k >> 1, r = k & 1;
        const float *xp = xb + 2 + q + r;
        vs[k] = snake(up_phase(tp, r, xp[0], xp[1], xp[2], xp[3], xp[4], xp[5]), a, inv_b);
      }
    } else {
      // edge tiles: clamp m into [0, 2T - 1] and take v there
      for (int k = tid; k < 2 * TILE + 12; k += THREADS) {
        int m = 2 * t0 - 6 + k;
        m = m < 0 ? 0 : (m > 2 * T - 1 ? 2 * T - 1 : m);
        const int p = m >> 1, r = m & 1;
        // x[p + r - 3 + k'] sits at xb[p + r - 3 + k' - (t0 - 8)]
        const float *xp = xb + (p + r + 5 - t0);
        vs[k] = snake(up_phase(tp, r, xp[0], xp[1], xp[2], xp[3], xp[4], xp[5]), a, inv_b);
      }
    }
    __syncthreads();

    // ---- stage B: y[t] = sum_j f_dn[j] v[2t + j - 5]; v[2t + j - 5] is vs[2 (t - t0) + j + 1]
    const int tl = 4 * tid;
    const float4 a0 = *reinterpret_cast<const float4 *>(vs + 2 * tl);
    const float4 a1 = *reinterpret_cast<const float4 *>(vs + 2 * tl + 4);
    const float4 a2 = *reinterpret_cast<const float4 *>(vs + 2 * tl + 8);
    const float4 a3 = *reinterpret_cast<const float4 *>(vs + 2 * tl + 12);
    const float4 a4 = *reinterpret_cast<const float4 *>(vs + 2 * tl + 16);
    const float vw[20] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w, a2.x, a2.y,
                          a2.z, a2.w, a3.x, a3.y, a3.z, a3.w, a4.x, a4.y, a4.z, a4.w};
    float out[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float acc = 0.0f;
#pragma unroll
      for (int j = 0; j < 12; ++j) acc = fmaf(tp.dn[j], vw[2 * e + j + 1], acc);
      out[e] = acc;
    }
    float *yr = y + row * (long long)T;
    const int t = t0 + tl;
    if (t + 3 < T && ((reinterpret_cast<uintptr_t>(yr + t) & 15u) == 0)) {
      __stcs(reinterpret_cast<float4 *>(yr + t), make_float4(out[0], out[1], out[2], out[3]));
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (t + e < T) yr[t + e] = out[e];
    }
  }
  cp_async_wait<0>();
}

__global__ void sin_squared_kernel(const float *__restrict__ z, float *__restrict__ out,
                                   long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    out[i] = sin_squared(z[i]);
}

// CTAs that are resident at once for the activation kernel on this device.
int persistent_ctas() {
  static int n = 0;
  if (n == 0) {
    int dev = 0, sms = 148, per_sm = 4;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, activation_kernel, THREADS, 0) !=
            cudaSuccess ||
        per_sm < 1)
      per_sm = 4;
    n = sms * per_sm;
  }
  return n;
}

}  // namespace

bv_status launch_sin_squared(const float *z, float *out, long long n, cudaStream_t st) {
  if (n <= 0) return BV_OK;
  const long long blocks = (n + 255) / 256;
  sin_squared_kernel<<<(unsigned)(blocks < 148 * 16 ? blocks : 148 * 16), 256, 0, st>>>(z, out,
                                                                                        n);
  count_launch();
  return check_launch("sin_squared_kernel");
}

bv_status launch_activation(const float *x, float *y, int B, int C, int T, const float *la,
                            const float *lb, const float *fu, const float *fd, float eps,
                            cudaStream_t st) {
  const long long rows = (long long)B * C;
  const int tiles = (T + TILE - 1) / TILE;
  const long long n_tiles = rows * tiles;
  if (n_tiles <= 0) return BV_OK;
  const int ctas = persistent_ctas();
  const long long grid = n_tiles < ctas ? n_tiles : ctas;
  {
    LaunchTimer tm(st, "activation", 0.0, 8.0 * (double)rows * T);
    activation_kernel<<<(unsigned)grid, THREADS, 0, st>>>(x, y, C, T, tiles, n_tiles, la, lb,
                                                          fu, fd, eps);
  }
  count_launch();
  return check_launch("activation_kernel");
}

}  // namespace bv
