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
// streams into the other half of a double buffer with cp.async.  Per tile,
// stage A computes v[2 t0 - 6 + k], k < 2 TILE + 12, into shared memory and
// stage B filters v into the TILE outputs.  Each thread works on two
// positions half a tile apart at once, with packed f32x2 arithmetic (FFMA2):
// both positions have the same polyphase taps, so every filter tap and every
// step of the sin^2 evaluation is one paired instruction.
#include <type_traits>

#include "common.cuh"
#include "sin2.cuh"

namespace bv {
namespace {

constexpr int TILE = 2048;         // outputs per tile
constexpr int HALF = TILE / 2;     // the two positions of a thread are HALF apart
constexpr int THREADS = 256;       // per half tile: 4 outputs and 8 up-sampled values each
constexpr int XS = TILE + 16;      // x[t0 - 8 + i]
// v[2 t0 - 6 + k], k < 2 TILE + 12, stored at vidx(k): 4 floats of padding
// after every 32 spread the 32-byte-strided float4 accesses of a warp over all
// banks
__device__ __forceinline__ int vidx(int k) { return k + 4 * (k >> 5); }
constexpr int VS = (2 * TILE + 16) + 4 * ((2 * TILE + 16) / 32 + 1);
static_assert(HALF == 4 * THREADS, "one thread per 4 outputs of a half tile");

__device__ __forceinline__ float2 f2(float v) { return make_float2(v, v); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }

// Scalar SnakeBeta (tails and edge fix-ups).
__device__ __forceinline__ float snake1(float u, float a, float inv_b) {
  return fmaf(sin_squared(a * u), inv_b, u);
}

// Paired SnakeBeta: u + sin^2(a u) inv_b for two values, with the sin^2 of
// sin2.cuh (reduction by pi in three parts, Taylor series of sin to r^13).
// The nearest integer to z/pi comes from adding and removing 1.5 * 2^23.
// CHECK = false when the caller has bounded |a u| by the fast-path limit.
template <bool CHECK = true>
__device__ __forceinline__ float2 snake2(float2 u, float a, float inv_b) {
  using namespace sin2c;
  const float2 z = mul2(u, f2(a));
  if (CHECK && fmaxf(fabsf(z.x), fabsf(z.y)) > kFastLimit)
    return make_float2(snake1(u.x, a, inv_b), snake1(u.y, a, inv_b));
  const float2 k = add2(fma2(z, f2(kInvPi), f2(12582912.0f)), f2(-12582912.0f));
  float2 r = fma2(k, f2(-kC1), z);
  r = fma2(k, f2(-kC2), r);
  r = fma2(k, f2(-kC3), r);
  const float2 r2 = mul2(r, r);
  float2 p = fma2(r2, f2(kT6), f2(kT5));
  p = fma2(r2, p, f2(kT4));
  p = fma2(r2, p, f2(kT3));
  p = fma2(r2, p, f2(kT2));
  p = fma2(r2, p, f2(kT1));
  p = fma2(r2, p, f2(1.0f));
  const float2 s = mul2(r, p);
  return fma2(mul2(s, s), f2(inv_b), u);
}

struct Taps {
  float up2[12];  // 2 * f_up
  float dn[12];
};

// u at phase r (0: even index, 1: odd) from six consecutive x values
// xp[0..5] = x[p + r - 3 .. p + r + 2]:  u[2p+r] = sum_l 2 f[2l+1-r] x[p+2+r-l],
// where term l pairs with xp[5-l].  (The phase is a template argument so the
// taps are indexed statically and stay in registers.)
template <int R>
__device__ __forceinline__ float up1r(const Taps &tp, const float *xp) {
  float u = tp.up2[1 - R] * xp[5];
#pragma unroll
  for (int l = 1; l < 6; ++l) u = fmaf(tp.up2[2 * l + 1 - R], xp[5 - l], u);
  return u;
}
__device__ __forceinline__ float up1(const Taps &tp, int r, const float *xp) {
  return r ? up1r<1>(tp, xp) : up1r<0>(tp, xp);
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

// Issue the copies of one tile's input into xs: x[t0 - 8 + i], clamped.
__device__ __forceinline__ void issue_tile(const float *__restrict__ xr, float *xs, int t0, int T,
                                           int tid) {
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

__device__ __forceinline__ void store4(float *yr, int t, int T, float o0, float o1, float o2,
                                       float o3) {
  if (t + 3 < T && ((reinterpret_cast<uintptr_t>(yr + t) & 15u) == 0)) {
    __stcs(reinterpret_cast<float4 *>(yr + t), make_float4(o0, o1, o2, o3));
  } else {
    if (t < T) yr[t] = o0;
    if (t + 1 < T) yr[t + 1] = o1;
    if (t + 2 < T) yr[t + 2] = o2;
    if (t + 3 < T) yr[t + 3] = o3;
  }
}

__global__ void __launch_bounds__(THREADS, 2)
activation_kernel(const float *__restrict__ x, float *__restrict__ y, int C, int T,
                  int tiles_per_row, int n_tiles, const float *__restrict__ log_alpha,
                  const float *__restrict__ log_beta, const float *__restrict__ f_up,
                  const float *__restrict__ f_dn, float eps) {
  __shared__ __align__(16) float xs[2][XS];
  __shared__ __align__(16) float vs[VS];
  __shared__ float snake_ab[2];  // a, inv_b of the current tile's channel
  const int tid = threadIdx.x;

  Taps tp;
#pragma unroll
  for (int j = 0; j < 12; ++j) {
    tp.up2[j] = 2.0f * __ldg(f_up + j);
    tp.dn[j] = __ldg(f_dn + j);
  }
  // the taps as broadcast pairs, formed once for every tile
  float2 U2[12], D2[12];
#pragma unroll
  for (int j = 0; j < 12; ++j) {
    U2[j] = f2(tp.up2[j]);
    D2[j] = f2(tp.dn[j]);
  }
  // |u| <= up_abs * max |x| over the six inputs of either phase
  float up_abs = 0.0f, up_abs1 = 0.0f;
#pragma unroll
  for (int l = 0; l < 6; ++l) {
    up_abs += fabsf(tp.up2[2 * l + 1]);
    up_abs1 += fabsf(tp.up2[2 * l]);
  }
  up_abs = fmaxf(up_abs, up_abs1);

  // tiles are visited as tile_id = blockIdx.x + k gridDim.x; (row, tile) are
  // carried along incrementally
  const int step_row = gridDim.x / tiles_per_row, step_tile = gridDim.x % tiles_per_row;
  int tile_id = blockIdx.x;
  int row = tile_id / tiles_per_row, tile = tile_id % tiles_per_row;
  if (tile_id < n_tiles) issue_tile(x + (size_t)row * T, xs[0], tile * TILE, T, tid);
  cp_async_commit();
  int buf = 0;
  for (; tile_id < n_tiles; tile_id += gridDim.x, buf ^= 1) {
    int nrow = row + step_row, ntile = tile + step_tile;
    if (ntile >= tiles_per_row) {
      ntile -= tiles_per_row;
      ++nrow;
    }
    if (tile_id + (int)gridDim.x < n_tiles)
      issue_tile(x + (size_t)nrow * T, xs[buf ^ 1], ntile * TILE, T, tid);
    cp_async_commit();
    if (tid == 0) {
      const int c = row % C;
      snake_ab[0] = expf(__ldg(log_alpha + c));
      snake_ab[1] = 1.0f / (expf(__ldg(log_beta + c)) + eps);
    }
    cp_async_wait<1>();  // this tile's copies are done; the next tile's may be in flight
    __syncthreads();

    const int t0 = tile * TILE;
    const float a = snake_ab[0], inv_b = snake_ab[1];
    const float *xb = xs[buf];

    // ---- stage A: v[2 t0 - 6 + k]; k = 2q + r holds p = t0 - 3 + q and
    // x[p + r - 3 + k'] sits at xb[2 + q + r + k'].  The thread owns
    // q in [4 tid, 4 tid + 4) of each half tile.
    {
      const int q0 = 4 * tid;
      float2 X[12];
#pragma unroll
      for (int w = 0; w < 3; ++w) {
        const float4 lo = *reinterpret_cast<const float4 *>(xb + q0 + 4 * w);
        const float4 hi = *reinterpret_cast<const float4 *>(xb + HALF + q0 + 4 * w);
        X[4 * w] = make_float2(lo.x, hi.x);
        X[4 * w + 1] = make_float2(lo.y, hi.y);
        X[4 * w + 2] = make_float2(lo.z, hi.z);
        X[4 * w + 3] = make_float2(lo.w, hi.w);
      }
      // every u of this thread is bounded by up_abs times its largest input:
      // when a times that bound is within sin^2's fast-path limit, the
      // per-pair range check is skipped (thread-uniform branch)
      float m = 0.0f;
#pragma unroll
      for (int j = 0; j < 12; ++j) m = fmaxf(m, fmaxf(fabsf(X[j].x), fabsf(X[j].y)));
      const bool fast = a * (up_abs * m) <= sin2c::kFastLimit;
      float2 V[8];
      auto stage_a = [&](auto check) {
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int b0 = 2 + qq + r;
            float2 u = mul2(U2[1 - r], X[b0 + 5]);
#pragma unroll
            for (int l = 1; l < 6; ++l) u = fma2(U2[2 * l + 1 - r], X[b0 + 5 - l], u);
            V[2 * qq + r] = snake2<decltype(check)::value>(u, a, inv_b);
          }
        }
      };
      if (fast)
        stage_a(std::false_type{});
      else
        stage_a(std::true_type{});
      *reinterpret_cast<float4 *>(vs + vidx(2 * q0)) = make_float4(V[0].x, V[1].x, V[2].x, V[3].x);
      *reinterpret_cast<float4 *>(vs + vidx(2 * q0 + 4)) =
          make_float4(V[4].x, V[5].x, V[6].x, V[7].x);
      *reinterpret_cast<float4 *>(vs + vidx(2 * HALF + 2 * q0)) =
          make_float4(V[0].y, V[1].y, V[2].y, V[3].y);
      *reinterpret_cast<float4 *>(vs + vidx(2 * HALF + 2 * q0 + 4)) =
          make_float4(V[4].y, V[5].y, V[6].y, V[7].y);
      // k in [2 TILE, 2 TILE + 12): one or two per warp, lane 0 and lane 1
      if ((tid & 31) < 2 && (tid >> 5) + 8 * (tid & 31) < 12) {
        const int i = (tid >> 5) + 8 * (tid & 31);
        const int k = 2 * TILE + i;
        const int q = k >> 1, r = k & 1;
        vs[vidx(k)] = snake1(up1(tp, r, xb + 2 + q + r), a, inv_b);
      }
    }
    // Near a row end the pages pad the 2x signal by replication: v at an index
    // m outside [0, 2T-1] is v at the clamped index.  Only m in [-6, -1] and
    // [2T, 2T + 4] are read by outputs t < T.
    const bool edge = (2 * t0 - 6 < 0) || (2 * t0 + 2 * TILE + 5 > 2 * T - 1);
    if (edge) {
      __syncthreads();
      if (tid < 11) {
        const int m = tid < 6 ? tid - 6 : 2 * T + (tid - 6);
        const int k = m - (2 * t0 - 6);
        if (k >= 0 && k < 2 * TILE + 12) {
          const int mc = m < 0 ? 0 : 2 * T - 1;
          const int p = mc >> 1, r = mc & 1;
          // x[p + r - 3 + k'] sits at xb[p + r + 5 - t0 + k'] (in range: the tile
          // reaches that row end)
          vs[vidx(k)] = snake1(up1(tp, r, xb + (p + r + 5 - t0)), a, inv_b);
        }
      }
    }
    __syncthreads();

    // ---- stage B: y[t] = sum_j f_dn[j] v[2t + j - 5]; v[2t + j - 5] is vs[2 (t - t0) + j + 1]
    {
      const int tl = 4 * tid;
      float2 W[20];
#pragma unroll
      for (int w = 0; w < 5; ++w) {
        const float4 lo = *reinterpret_cast<const float4 *>(vs + vidx(2 * tl + 4 * w));
        const float4 hi = *reinterpret_cast<const float4 *>(vs + vidx(2 * HALF + 2 * tl + 4 * w));
        W[4 * w] = make_float2(lo.x, hi.x);
        W[4 * w + 1] = make_float2(lo.y, hi.y);
        W[4 * w + 2] = make_float2(lo.z, hi.z);
        W[4 * w + 3] = make_float2(lo.w, hi.w);
      }
      float2 out[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 acc = mul2(D2[0], W[2 * e + 1]);
#pragma unroll
        for (int j = 1; j < 12; ++j) acc = fma2(D2[j], W[2 * e + j + 1], acc);
        out[e] = acc;
      }
      float *yr = y + (size_t)row * T;
      store4(yr, t0 + tl, T, out[0].x, out[1].x, out[2].x, out[3].x);
      store4(yr, t0 + HALF + tl, T, out[0].y, out[1].y, out[2].y, out[3].y);
    }
    row = nrow;
    tile = ntile;
  }
  cp_async_wait<0>();
}

__global__ void sin_squared_kernel(const float *__restrict__ z, float *__restrict__ out,
                                   long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    out[i] = sin_squared(z[i]);
}

// CTAs resident at once for the activation kernel on this device.
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
  if (n_tiles > 0x7fffffffLL) return fail(BV_ERR_SHAPE, "activation: too many tiles");
  const int ctas = persistent_ctas();
  const long long grid = n_tiles < ctas ? n_tiles : ctas;
  {
    LaunchTimer tm(st, "activation", 0.0, 8.0 * (double)rows * T);
    activation_kernel<<<(unsigned)grid, THREADS, 0, st>>>(x, y, C, T, tiles, (int)n_tiles, la,
                                                          lb, fu, fd, eps);
  }
  count_launch();
  return check_launch("activation_kernel");
}

}  // namespace bv
