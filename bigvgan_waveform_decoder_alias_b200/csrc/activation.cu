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
// Work unit: a warp tile, TW outputs of two rows at once (rows r0 and r0 + 1;
// channels may differ).  Everything in shared memory is stored as (row r0,
// row r0 + 1) pairs, so every load yields operand pairs for packed f32x2
// arithmetic (FFMA2) directly: the two rows share the filter taps, and their
// SnakeBeta constants sit in pairs too.
//
// Every warp runs on its own, with no block-wide barrier: it owns a
// contiguous range of warp tiles (row pair by row pair, left to right) and
// its own shared memory -- a double buffer of input windows, filled with
// cp.async one tile ahead, and two 2x-rate buffers.  Stage A of tile j
// computes v[2 t0 - 5 + s], s < 2 TW, into its buffer; stage B of tile j also
// needs the first 10 values of tile j + 1 (slots 2 TW .. 2 TW + 9), so it runs
// after stage A of tile j + 1, which writes those values into both buffers.
// Only at the end of a row (replicate padding) or of the warp's range does
// stage B follow its own stage A, after computing those 10 values directly.
//
// SnakeBeta's sin^2 runs in units of pi: w = u a/pi, f = w - rint(w) in
// [-1/2, 1/2] (exact), and sin(pi f) = f P(f^2) with a degree-4 polynomial P
// (sin2.cuh).  The row's sqrt(inv_b) is folded into P, so v = u + g^2 with
// g = f P'(f^2): eleven paired instructions per pair of values.
#include <atomic>
#include <type_traits>

#include "common.cuh"
#include "sin2.cuh"

namespace bv {
namespace {

constexpr int WARPS = 8;          // per CTA
constexpr int THREADS = 32 * WARPS;
constexpr int TW = 128;           // outputs per row of a warp tile (4 per lane)
constexpr int XP = TW + 16;       // input pairs x[t0 - 8 + i] of a warp tile
constexpr int VP = 2 * TW + 10;   // 2x-rate pairs v[2 t0 - 5 + s] of a warp tile

// Shared-memory float offsets of pair i.  A 16-byte chunk c holds two pairs;
// the chunks are padded so that the 16-byte accesses of a quarter warp hit 8
// distinct bank groups while the address stays linear in the lane:
//   input pairs: stage A's lanes are 2 chunks apart; chunk c at c + c/2,
//     so lane L's chunks start at 3L (3L mod 8 distinct over 8 lanes);
//   2x-rate pairs: stages A and B have lanes 4 chunks apart; chunk c at
//     c + c/4, lane L's chunks start at 5L.
__host__ __device__ constexpr int xoff(int i) { return 4 * ((i >> 1) + (i >> 2)) + 2 * (i & 1); }
__host__ __device__ constexpr int voff(int s) { return 4 * ((s >> 1) + (s >> 3)) + 2 * (s & 1); }
constexpr int XS_FLOATS = xoff(XP - 1) + 2;
constexpr int VS_FLOATS = voff(VP - 1) + 2;
// Per warp: NX input windows (a ring, filled NX - 1 tiles ahead), two 2x-rate
// buffers and the row pair's SnakeBeta constants.
__host__ __device__ constexpr int warp_floats(int nx) { return nx * XS_FLOATS + 2 * VS_FLOATS + 2 * 10; }
constexpr int K1_NX = 2;  // input windows of activation_kernel
constexpr int WARP_FLOATS = warp_floats(K1_NX);
constexpr size_t SMEM_BYTES = (size_t)WARPS * WARP_FLOATS * sizeof(float);
static_assert(TW == 4 * 32, "4 outputs per lane");
static_assert(XS_FLOATS % 4 == 0 && VS_FLOATS % 4 == 0 && WARP_FLOATS % 4 == 0, "16-byte alignment");
static_assert(xoff(32) == xoff(0) + 96 && voff(2 * TW) == 640, "linear layouts");

// |w| bound of the fast path: far inside the 2^22 where rint by adding and
// removing 1.5 * 2^23 stays exact; |a u| <= pi * 16384 = 51472.
constexpr float kWLimit = 16384.0f;

// Per-row-pair constants, as (row r0, row r0 + 1) pairs.
enum {
  kA = 0,      // a / pi
  kP = 1,      // P_j sqrt(inv_b), j < 5
  kM = 6,      // 1.5 * 2^23 (both)
  kNeg = 7,    // -1 (both)
  kAraw = 8,   // a
  kIb = 9,     // inv_b
  kConsts = 10
};

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }

struct Snake {
  float2 A, P[5], M, Neg;
};

__device__ __forceinline__ void load_snake(Snake &k, const float2 *cst) {
  const float4 *c4 = reinterpret_cast<const float4 *>(cst);
  float4 v = c4[0];
  k.A = make_float2(v.x, v.y);
  k.P[0] = make_float2(v.z, v.w);
  v = c4[1];
  k.P[1] = make_float2(v.x, v.y);
  k.P[2] = make_float2(v.z, v.w);
  v = c4[2];
  k.P[3] = make_float2(v.x, v.y);
  k.P[4] = make_float2(v.z, v.w);
  v = c4[3];
  k.M = make_float2(v.x, v.y);
  k.Neg = make_float2(v.z, v.w);
}

// Paired SnakeBeta for the two rows.  CHECK: range-check |w| per pair and
// take the scalar sin^2 of sin2.cuh (Cody-Waite reduction, sinf beyond its
// limit) for pairs outside the fast path.
template <bool CHECK>
__device__ __forceinline__ float2 snake2(float2 u, const Snake &k, const float2 *cst) {
  const float2 w = mul2(u, k.A);
  if (CHECK && fmaxf(fabsf(w.x), fabsf(w.y)) > kWLimit) {
    const float2 a = cst[kAraw], ib = cst[kIb];
    return make_float2(fmaf(sin_squared(a.x * u.x), ib.x, u.x),
                       fmaf(sin_squared(a.y * u.y), ib.y, u.y));
  }
  const float2 t = add2(w, k.M);          // rint(w) + 1.5 * 2^23
  const float2 nk = fma2(t, k.Neg, k.M);  // -rint(w), exact
  const float2 f = add2(w, nk);           // in [-1/2, 1/2], exact
  const float2 s = mul2(f, f);
  float2 p = fma2(s, k.P[4], k.P[3]);
  p = fma2(s, p, k.P[2]);
  p = fma2(s, p, k.P[1]);
  p = fma2(s, p, k.P[0]);
  const float2 g = mul2(f, p);  // sqrt(inv_b) sin(pi f)
  return fma2(g, g, u);
}

// u pair at phase R from six consecutive input pairs xp[0..5] =
// x[p + R - 3 .. p + R + 2]: u[2p+R] = sum_l 2 f_up[2l+1-R] x[p+2+R-l], term l
// pairs with xp[5-l].
template <int R>
__device__ __forceinline__ float2 up2(const float2 *U2, const float2 *xp) {
  float2 u = mul2(U2[1 - R], xp[5]);
#pragma unroll
  for (int l = 1; l < 6; ++l) u = fma2(U2[2 * l + 1 - R], xp[5 - l], u);
  return u;
}

__device__ __forceinline__ void cp_async4(float *dst, const float *src) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Issue the copies of one warp tile's input: pair i = (x0[t0 - 8 + i],
// x1[t0 - 8 + i]), positions clamped to [0, T).  Lane L copies pairs L + 32 j
// of each row (j < 5, the last only for L < 16).
__device__ __forceinline__ void issue_tile(const float *__restrict__ x0,
                                           const float *__restrict__ x1, float *xs, int t0, int T,
                                           int lane) {
  float *d = xs + xoff(lane);  // xoff(L + 32 j) = xoff(L) + 96 j
  const int base = t0 - 8 + lane;
  if (t0 >= 8 && t0 - 8 + XP <= T) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      cp_async4(d + 96 * j, x0 + base + 32 * j);
      cp_async4(d + 96 * j + 1, x1 + base + 32 * j);
    }
    if (lane < XP - 128) {
      cp_async4(d + 384, x0 + base + 128);
      cp_async4(d + 385, x1 + base + 128);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 5; ++j) {
      if (j < 4 || lane < XP - 128) {
        int p = base + 32 * j;
        p = p < 0 ? 0 : (p > T - 1 ? T - 1 : p);
        cp_async4(d + 96 * j, x0 + p);
        cp_async4(d + 96 * j + 1, x1 + p);
      }
    }
  }
}

// Four consecutive outputs: one 16-byte store where the row allows it, two
// 8-byte stores where it is only 8-byte aligned (rows of an even length not a
// multiple of 4 alternate between the two), else four 4-byte stores.
__device__ __forceinline__ void store4(float *yr, int t, int T, float o0, float o1, float o2,
                                       float o3) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(yr + t);
  if (t + 3 < T && (a & 15u) == 0) {
    __stcs(reinterpret_cast<float4 *>(yr + t), make_float4(o0, o1, o2, o3));
  } else if (t + 3 < T && (a & 7u) == 0) {
    __stcs(reinterpret_cast<float2 *>(yr + t), make_float2(o0, o1));
    __stcs(reinterpret_cast<float2 *>(yr + t + 2), make_float2(o2, o3));
  } else {
    if (t < T) yr[t] = o0;
    if (t + 1 < T) yr[t + 1] = o1;
    if (t + 2 < T) yr[t + 2] = o2;
    if (t + 3 < T) yr[t + 3] = o3;
  }
}

__device__ __forceinline__ void load_taps(float2 (&F)[12], const float2 *taps) {
#pragma unroll
  for (int j = 0; j < 6; ++j) {
    const float4 v = reinterpret_cast<const float4 *>(taps)[j];
    F[2 * j] = make_float2(v.x, v.y);
    F[2 * j + 1] = make_float2(v.z, v.w);
  }
}

// Stage A of one warp tile: lane L's 2x-rate pairs s = 8 L + n, n < 8, i.e.
// k = s + 1 = 2q + r from (q0, 1) to (q0 + 4, 0) with q0 = 4 L relative to
// t0 - 3; their inputs are the pairs q0 + 3 .. q0 + 11 (X[j] = pair q0 + 2 + j,
// whose chunks start at 3 L + 1 in the padded layout).  The slots s < 10 are
// written to the other buffer's slots s + 2 TW too (mirror), where the
// previous tile's stage B reads them.
// TAIL: lanes 0-9 also compute the 10 pairs past the tile's end from its own
// window (as stage_a_tail does), with the taps and constants already loaded.
template <bool TAIL = false>
__device__ __forceinline__ void stage_a(const float *xb, float *vb, float *vmirror,
                                        const float2 *taps, const float2 *cst, float up_abs,
                                        int lane) {
  float2 U2[12];
  load_taps(U2, taps);
  Snake k;
  load_snake(k, cst);
  float2 X[10];
  const float *xl = xb + 12 * lane;  // xoff(4L + 2 + 2m) = 12 L + 4 (1 + m + (1 + m) / 2)
#pragma unroll
  for (int m = 0; m < 5; ++m) {
    const float4 v = *reinterpret_cast<const float4 *>(xl + 4 * (1 + m + (1 + m) / 2));
    X[2 * m] = make_float2(v.x, v.y);
    X[2 * m + 1] = make_float2(v.z, v.w);
  }
  // every u of this lane is bounded by up_abs times its largest input: when
  // that keeps |w| within the fast path, the per-pair range check is skipped
  // (lane-uniform branch)
  float mx = 0.0f;
#pragma unroll
  for (int j = 1; j < 10; ++j) mx = fmaxf(mx, fmaxf(fabsf(X[j].x), fabsf(X[j].y)));
  float *vl = vb + 20 * lane;  // voff(8L + n) = 20 L + 2n
  auto run = [&](auto check) {
    constexpr bool CK = decltype(check)::value;
#pragma unroll
    for (int n = 0; n < 8; n += 2) {
      // n (even): phase 1 at q0 + n/2; n + 1: phase 0 at q0 + n/2 + 1; both
      // read the input pairs X[n/2 + 1 ..]
      const float2 v0 = snake2<CK>(up2<1>(U2, X + n / 2 + 1), k, cst);
      const float2 v1 = snake2<CK>(up2<0>(U2, X + n / 2 + 1), k, cst);
      const float4 o = make_float4(v0.x, v0.y, v1.x, v1.y);
      *reinterpret_cast<float4 *>(vl + 2 * n) = o;
      if (vmirror && 8 * lane + n < 10)
        *reinterpret_cast<float4 *>(vmirror + voff(8 * lane + n + 2 * TW)) = o;
    }
  };
  if (mx * up_abs * fmaxf(k.A.x, k.A.y) <= kWLimit)
    run(std::false_type{});
  else
    run(std::true_type{});
  if (TAIL && lane < 10) {
    // pair s = 2 TW + i, i = lane: lanes 0-4 phase 1 at q = TW + L, lanes
    // 5-9 phase 0 at q = TW + L - 4 (the layout of stage_a_tail)
    const int R = lane < 5 ? 1 : 0;
    const int q = lane < 5 ? TW + lane : TW + lane - 4;
    float2 xp[6];
#pragma unroll
    for (int j = 0; j < 6; ++j) xp[j] = *reinterpret_cast<const float2 *>(xb + xoff(2 + q + R + j));
    const float2 u = R ? up2<1>(U2, xp) : up2<0>(U2, xp);
    *reinterpret_cast<float2 *>(vb + voff(2 * q + R - 1)) = snake2<true>(u, k, cst);
  }
}

// The 10 pairs s in [2 TW, 2 TW + 10) of a tile, from its own input window:
// k = s + 1 = 2 TW + 1 + i; lanes 0-4 take phase 1 (q = TW + L), lanes 5-9
// phase 0 (q = TW + L - 4).
__device__ __forceinline__ void stage_a_tail(const float *xb, float *vb, const float2 *taps,
                                             const float2 *cst, int lane) {
  if (lane >= 10) return;
  float2 U2[12];
  load_taps(U2, taps);
  Snake k;
  load_snake(k, cst);
  const int R = lane < 5 ? 1 : 0;
  const int q = lane < 5 ? TW + lane : TW + lane - 4;
  float2 xp[6];
#pragma unroll
  for (int j = 0; j < 6; ++j) xp[j] = *reinterpret_cast<const float2 *>(xb + xoff(2 + q + R + j));
  const float2 u = R ? up2<1>(U2, xp) : up2<0>(U2, xp);
  *reinterpret_cast<float2 *>(vb + voff(2 * q + R - 1)) = snake2<true>(u, k, cst);
}

// Stage B of one warp tile: y[t] = sum_j f_dn[j] v[2t + j - 5] with
// v[2t + j - 5] at s = 2 (t - t0) + j; lane L writes t = t0 + 4 L + e.
__device__ __forceinline__ void stage_b(const float *vb, const float2 *taps, float *y0,
                                        bool has_r1, int t0, int T, int lane) {
  float2 D2[12];
  load_taps(D2, taps + 12);
  float2 W[18];
  const float *vl = vb + 20 * lane;  // voff(8L + 2m) = 20 L + 4 (m + m / 4)
#pragma unroll
  for (int m = 0; m < 9; ++m) {
    const float4 v = *reinterpret_cast<const float4 *>(vl + 4 * (m + m / 4));
    W[2 * m] = make_float2(v.x, v.y);
    W[2 * m + 1] = make_float2(v.z, v.w);
  }
  float2 out[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float2 acc = mul2(D2[0], W[2 * e]);
#pragma unroll
    for (int j = 1; j < 12; ++j) acc = fma2(D2[j], W[2 * e + j], acc);
    out[e] = acc;
  }
  const int t = t0 + 4 * lane;
  store4(y0, t, T, out[0].x, out[1].x, out[2].x, out[3].x);
  if (has_r1) store4(y0 + T, t, T, out[0].y, out[1].y, out[2].y, out[3].y);
}

__device__ __forceinline__ void copy_pair(float *vb, int dst, int src) {
  *reinterpret_cast<float2 *>(vb + voff(dst)) = *reinterpret_cast<const float2 *>(vb + voff(src));
}

// ---------------------------------------------------------------------------
// The same activation writing the operand planes of the time-major
// tensor-core conv instead of [B, C, T]: hi[b, t, c] = tf32(y[b, c, t]) and
// lo = y - hi, so the activation's output never exists in [B, C, T] form and
// no separate transpose pass reads it back.
//
// A team of TW_ warps owns a contiguous range of tasks (a group of 2 TW_
// channels of one batch row, time tile), group-major; warp k of the team
// takes the group's row pair k (channels 2k, 2k + 1) and walks the range's
// tiles exactly as activation_kernel walks a row pair, so consecutive tiles
// share their 2x-rate values and the SnakeBeta constants are set up once per
// row pair.  Stage B writes the pair's TW outputs into the team's staging
// buffer, one region per row pair (time steps as (channel 2k, 2k + 1)
// pairs); after a named barrier over the team each warp writes its share of
// the tile's time steps, all 2 TW_ channels of each, to both planes.  Two
// staging buffers alternate, so one barrier per tile orders both the writes
// before the flush and the flush before the buffer's next use.
//
// The flush is what costs: a 16-byte store instruction whose 32 lanes write
// pieces of many cache lines is paid per line on the SM's write path (with
// only the hi plane written the kernel ran in 0.65 of the time).  Three team
// shapes, the widest the channel count allows:
//   32 channels (C a multiple of 32): one team of 16 warps per CTA; eight
//     lanes write one time step's 32 channels, a whole aligned 128-byte line
//     of each plane, four lines per instruction;
//   16 channels: one team of 8 warps per CTA; 64 bytes, 8 lines;
//   8 channels: two teams of 4 warps per CTA; 32 bytes, 16 lines.
template <int TW_>
struct TeamShape {
  static constexpr int kWarps = TW_;                  // per team = row pairs per group
  static constexpr int kCh = 2 * TW_;                 // channels per group
  static constexpr int kCtaWarps = TW_ < WARPS ? WARPS : TW_;
  static constexpr int kTeams = kCtaWarps / TW_;
  static constexpr int kLanesPerStep = TW_ / 2;       // lanes per time step in the flush
  static constexpr int kStepsPerRound = 32 / kLanesPerStep;
  static constexpr int kStepsPerWarp = TW / TW_;      // of a tile's TW time steps
  // region r of a staging buffer: 16-byte aligned, and shifted by 64 / TW_
  // floats per region pair so that a half warp's 8-byte flush reads (32 / TW_
  // time steps of each of its TW_ / 2 region pairs) hit distinct banks
  __host__ __device__ static constexpr int region(int r) {
    return 2 * TW * r + (64 / TW_) * (r >> 1);
  }
  static constexpr int kStgFloats = (region(TW_ - 1) + 2 * TW + 3) / 4 * 4;
};
constexpr int TM_NX = 3;                // input windows per warp: two tiles in flight
constexpr int TM_WARP_FLOATS = warp_floats(TM_NX);
static_assert(TM_WARP_FLOATS % 4 == 0, "16-byte alignment");
template <int TW_>
constexpr size_t tm_smem_bytes() {
  using S = TeamShape<TW_>;
  return ((size_t)S::kCtaWarps * TM_WARP_FLOATS + (size_t)S::kTeams * 2 * S::kStgFloats) *
         sizeof(float);
}
static_assert(TeamShape<4>::kTeams == 2 && TeamShape<8>::kTeams == 1 &&
                  TeamShape<16>::kTeams == 1, "team shapes");
static_assert(TeamShape<4>::kStepsPerWarp == 2 * TeamShape<4>::kStepsPerRound &&
                  TeamShape<16>::kStepsPerWarp == 2 * TeamShape<16>::kStepsPerRound,
              "two flush rounds");
static_assert(tm_smem_bytes<16>() <= 227 * 1024 && 2 * tm_smem_bytes<8>() <= 228 * 1024 &&
                  2 * tm_smem_bytes<4>() <= 228 * 1024,
              "shared memory");

// Barrier 1 + team over the team's warps (immediate ids, so that the kernel
// reserves only the barriers it uses).
template <int TW_>
__device__ __forceinline__ void team_barrier(int team) {
  if constexpr (TeamShape<TW_>::kTeams == 1) {
    asm volatile("bar.sync 1, %0;\n" ::"n"(32 * TW_) : "memory");
  } else {
    static_assert(TeamShape<TW_>::kTeams == 2, "two teams");
    if (team == 0)
      asm volatile("bar.sync 1, %0;\n" ::"n"(32 * TW_) : "memory");
    else
      asm volatile("bar.sync 2, %0;\n" ::"n"(32 * TW_) : "memory");
  }
}

// Float offset of time step tl's (channel 2k, 2k + 1) pair in a staging
// region: 2 tl, with the two 16-byte chunks of every 32-byte lane slot
// swapped in the upper half of each 16-step block.
__device__ __forceinline__ int stg_index(int tl) { return (2 * tl) ^ (((tl >> 4) & 1) << 2); }

// Stage B of row pair k into its staging region: lane L holds t = 4 L + e,
// stored as (channel 2k, 2k + 1) pairs, two 16-byte stores per lane.
__device__ __forceinline__ void stage_b_stage(const float *vb, const float2 *taps, float *region,
                                              int lane) {
  float2 D2[12];
  load_taps(D2, taps + 12);
  float2 W[18];
  const float *vl = vb + 20 * lane;
#pragma unroll
  for (int m = 0; m < 9; ++m) {
    const float4 v = *reinterpret_cast<const float4 *>(vl + 4 * (m + m / 4));
    W[2 * m] = make_float2(v.x, v.y);
    W[2 * m + 1] = make_float2(v.z, v.w);
  }
  float2 out[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float2 acc = mul2(D2[0], W[2 * e]);
#pragma unroll
    for (int j = 1; j < 12; ++j) acc = fma2(D2[j], W[2 * e + j], acc);
    out[e] = acc;
  }
  // the two 16-byte chunks of lane L swap places when bit 2 of L is set
  // (stg_index), so each quarter warp's stores hit 8 distinct bank groups
  const int s = (lane >> 2) & 1;
  float4 *r4 = reinterpret_cast<float4 *>(region + 8 * lane);
  r4[s] = make_float4(out[0].x, out[0].y, out[1].x, out[1].y);
  r4[1 - s] = make_float4(out[2].x, out[2].y, out[3].x, out[3].y);
}

// Warp k's share of a staged tile: time steps kStepsPerWarp k .. + kStepsPerWarp
// - 1, per round kStepsPerRound time steps x the group's 4-channel quarters
// (kLanesPerStep lanes write one time step's row of a plane).  Quarter h's
// channels are the pairs of regions 2 h and 2 h + 1.
template <int TW_, bool F16>
__device__ __forceinline__ void flush_share(const float *sb, float *__restrict__ hi,
                                            float *__restrict__ lo, size_t obase, int C, int t0,
                                            int T, int k, int lane, float &vmax) {
  using S = TeamShape<TW_>;
  const int h = lane % S::kLanesPerStep;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int tl = S::kStepsPerWarp * k + S::kStepsPerRound * r + lane / S::kLanesPerStep;
    const int t = t0 + tl;
    const float2 a = *reinterpret_cast<const float2 *>(sb + S::region(2 * h) + stg_index(tl));
    const float2 c = *reinterpret_cast<const float2 *>(sb + S::region(2 * h + 1) + stg_index(tl));
    if (t < T) {
      const float v[4] = {a.x, a.y, c.x, c.y};
      const size_t o = obase + (size_t)t * C + 4 * h;
      if constexpr (F16) {
        // fp16 planes: hi = fp16(v), lo = fp16(v - hi), four channels in 8 bytes
        vmax = fmaxf(vmax, fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))));
        __half2 h2[2], l2[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          h2[q] = __floats2half2_rn(v[2 * q], v[2 * q + 1]);
          const float2 back = __half22float2(h2[q]);
          l2[q] = __floats2half2_rn(v[2 * q] - back.x, v[2 * q + 1] - back.y);
        }
        *reinterpret_cast<uint2 *>(reinterpret_cast<__half *>(hi) + o) =
            make_uint2(*reinterpret_cast<const unsigned *>(&h2[0]),
                       *reinterpret_cast<const unsigned *>(&h2[1]));
        *reinterpret_cast<uint2 *>(reinterpret_cast<__half *>(lo) + o) =
            make_uint2(*reinterpret_cast<const unsigned *>(&l2[0]),
                       *reinterpret_cast<const unsigned *>(&l2[1]));
      } else {
        float g[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) g[q] = __uint_as_float(__float_as_uint(v[q]) & 0xFFFFE000u);
        *reinterpret_cast<float4 *>(hi + o) = make_float4(g[0], g[1], g[2], g[3]);
        *reinterpret_cast<float4 *>(lo + o) =
            make_float4(v[0] - g[0], v[1] - g[1], v[2] - g[2], v[3] - g[3]);
      }
    }
  }
}

// The tile walk of both kernels.  TM = false: each warp owns a contiguous
// range of (row pair, tile) ids, row pair major, and writes y [rows, T].
// TM = true: each team owns a range of (8-channel group, tile) tasks and
// warp k walks row pair 4 group + k of them, writing the hi/lo planes
// [B, T, C] (y = hi).  NX input windows per warp: the copies of the next
// NX - 1 tiles are in flight while a tile is computed.  TW_: warps per team
// (TM), which also fixes the CTA's warps (TeamShape).
template <bool TM, int NX, int TW_ = 4, bool F16 = false>
__device__ __forceinline__ void activation_walk(
    const float *__restrict__ x, float *__restrict__ y, float *__restrict__ lo, int rows, int C,
    int T, int tiles_per_row, long long n_ids, const float *__restrict__ log_alpha,
    const float *__restrict__ log_beta, const float *__restrict__ f_up,
    const float *__restrict__ f_dn, float eps, int *status = nullptr) {
  extern __shared__ __align__(16) float smem[];
  __shared__ __align__(16) float2 taps[24];  // 2 f_up, then f_down, as broadcast pairs
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x < 24) {
    const float f =
        threadIdx.x < 12 ? 2.0f * __ldg(f_up + threadIdx.x) : __ldg(f_dn + threadIdx.x - 12);
    taps[threadIdx.x] = make_float2(f, f);
  }
  __syncthreads();  // the only block-wide barrier
  // |u| <= up_abs * max |x| over the six inputs of either phase
  float up_abs = 0.0f, up_abs1 = 0.0f;
#pragma unroll
  for (int l = 0; l < 6; ++l) {
    up_abs += fabsf(taps[2 * l + 1].x);
    up_abs1 += fabsf(taps[2 * l].x);
  }
  up_abs = fmaxf(up_abs, up_abs1);

  static_assert(NX >= 2 && NX <= 4, "input ring");
  constexpr int WF = warp_floats(NX);
  float *wsm = smem + (size_t)warp * WF;
  float *const xs0 = wsm, *const vs0 = wsm + NX * XS_FLOATS;  // buffer b at + b * size
  float2 *cst = reinterpret_cast<float2 *>(wsm + NX * XS_FLOATS + 2 * VS_FLOATS);
  using S = TeamShape<TW_>;
  constexpr int CTA_WARPS = TM ? S::kCtaWarps : WARPS;
  const int team = warp / S::kWarps, k = warp % S::kWarps;
  float *const stg = smem + (size_t)CTA_WARPS * WF + (size_t)team * 2 * S::kStgFloats;

  // this warp's (or team's) contiguous range of ids (row pair or group) *
  // tiles_per_row + tile
  const long long nw = (long long)gridDim.x * (TM ? S::kTeams : WARPS);
  const long long gw = (long long)blockIdx.x * (TM ? S::kTeams : WARPS) + (TM ? team : warp);
  const long long beg = gw * n_ids / nw, end = (gw + 1) * n_ids / nw;
  if (beg >= end) return;
  auto row_ptr = [&](int pr, int which) {
    const int r = 2 * pr + which;
    return x + (size_t)(r < rows ? r : rows - 1) * T;
  };
  constexpr int kStep = TM ? S::kWarps : 1;  // row pairs from one id row to the next
  int pair = (int)(beg / tiles_per_row), tile = (int)(beg % tiles_per_row);
  if (TM) pair = S::kWarps * pair + k;
  // (fpair, ftile): the tile of id fid = id + NX - 1, whose copies the
  // iteration of id issues; the prologue issues ids beg .. beg + NX - 2
  int fpair = pair, ftile = tile;
  long long fid = beg;
  auto advance = [&](int &pr, int &tl) {
    if (++tl == tiles_per_row) {
      tl = 0;
      pr += kStep;
    }
  };
#pragma unroll
  for (int j = 0; j < NX - 1; ++j) {
    if (fid < end) issue_tile(row_ptr(fpair, 0), row_ptr(fpair, 1), xs0 + j * XS_FLOATS,
                              ftile * TW, T, lane);
    cp_async_commit();
    ++fid;
    advance(fpair, ftile);
  }
  int xslot = 0;  // input window of id (id - beg mod NX)
  int cur_pair = -1;
  bool pending = false;  // stage B of the previous tile still to run
  int p_t0 = 0;
  size_t obase = 0;  // TM: plane offset of the group's (b, t = 0, first channel)
  int n_out = 0;     // TM: staged tiles so far (selects the staging buffer)
  float vmax = 0.0f;  // F16: the largest |value| written to the fp16 planes
  auto emit = [&](const float *vsrc, int t_out) {
    if constexpr (TM) {
      float *sb = stg + (n_out & 1) * S::kStgFloats;
      ++n_out;
      stage_b_stage(vsrc, taps, sb + S::region(k), lane);
      team_barrier<TW_>(team);
      flush_share<TW_, F16>(sb, y, lo, obase, C, t_out, T, k, lane, vmax);
    } else {
      stage_b(vsrc, taps, y + (size_t)(2 * pair) * T, 2 * pair + 1 < rows, t_out, T, lane);
    }
  };
  for (long long id = beg; id < end; ++id) {
    const int b = (int)((id - beg) & 1);
    int npair = pair, ntile = tile;
    advance(npair, ntile);
    __syncwarp();  // the previous iteration's reads of the buffers written below are done
    {
      // the window of id + NX - 1 is the one id - 1 used
      const int fslot = xslot == 0 ? NX - 1 : xslot - 1;
      if (fid < end)
        issue_tile(row_ptr(fpair, 0), row_ptr(fpair, 1), xs0 + fslot * XS_FLOATS, ftile * TW, T,
                   lane);
      cp_async_commit();
      ++fid;
      advance(fpair, ftile);
    }
    if (pair != cur_pair) {
      // the row pair's SnakeBeta constants (every lane computes the same values)
      cur_pair = pair;
      float *cf = reinterpret_cast<float *>(cst);
      const int r1 = min(2 * pair + 1, rows - 1);
      const int c0 = (2 * pair) % C, c1 = r1 % C;
      const float a0 = expf(__ldg(log_alpha + c0)), a1 = expf(__ldg(log_alpha + c1));
      const float ib0 = 1.0f / (expf(__ldg(log_beta + c0)) + eps);
      const float ib1 = 1.0f / (expf(__ldg(log_beta + c1)) + eps);
      const float sb0 = sqrtf(ib0), sb1 = sqrtf(ib1);
      if (lane == 0) {
        cf[2 * kA] = a0 * sin2p::kInvPi;
        cf[2 * kA + 1] = a1 * sin2p::kInvPi;
#pragma unroll
        for (int q = 0; q < 5; ++q) {
          cf[2 * (kP + q)] = sin2p::coef(q) * sb0;
          cf[2 * (kP + q) + 1] = sin2p::coef(q) * sb1;
        }
        cf[2 * kM] = cf[2 * kM + 1] = 12582912.0f;
        cf[2 * kNeg] = cf[2 * kNeg + 1] = -1.0f;
        cf[2 * kAraw] = a0;
        cf[2 * kAraw + 1] = a1;
        cf[2 * kIb] = ib0;
        cf[2 * kIb + 1] = ib1;
      }
      if (TM) {
        const int row0 = 2 * (pair - k), bb = row0 / C;
        obase = (size_t)bb * T * C + (row0 - bb * C);
      }
    }
    cp_async_wait<NX - 1>();  // this tile's input has landed (the next ones may be in flight)
    __syncwarp();
    const int t0 = tile * TW;
    const float *xb = xs0 + xslot * XS_FLOATS;
    xslot = xslot == NX - 1 ? 0 : xslot + 1;
    float *vb = vs0 + b * VS_FLOATS, *vo = vs0 + (b ^ 1) * VS_FLOATS;
    stage_a(xb, vb, vo, taps, cst, up_abs, lane);
    __syncwarp();
    // Replicate padding of the 2x signal: v[m] for m in [-5, -1] is v[0], for
    // m in [2T, 2T + 4] it is v[2T - 1] (slot s = m - 2 t0 + 5; only m up to
    // 2T + 4 are read).  The slots below 2 TW are fixed here (and mirrored,
    // below 10), before the previous tile's stage B reads the first 10.
    const bool row_end = tile == tiles_per_row - 1;
    const bool edge_r = T <= t0 + TW + 2;  // the tile's outputs read v[2T..]
    const int s_end = 2 * (T - t0) + 4;    // slot of v[2T - 1]
    if (t0 == 0 || edge_r) {
      if (lane < 5) {
        if (t0 == 0) copy_pair(vb, lane, 5);
        const int s = s_end + 1 + lane;
        if (edge_r && s < 2 * TW) {
          copy_pair(vb, s, s_end);
          if (s < 10)
            *reinterpret_cast<float2 *>(vo + voff(s + 2 * TW)) =
                *reinterpret_cast<const float2 *>(vb + voff(s_end));
        }
      }
      __syncwarp();
    }
    if (pending) emit(vo, p_t0);
    if (row_end || id + 1 == end) {
      // stage B of this tile now: its last 10 values come from its own window
      stage_a_tail(xb, vb, taps, cst, lane);
      __syncwarp();
      if (edge_r && lane < 5) {
        const int s = s_end + 1 + lane;
        if (s >= 2 * TW && s < VP) copy_pair(vb, s, s_end);
      }
      __syncwarp();
      emit(vb, t0);
      pending = false;
    } else {
      pending = true;
      p_t0 = t0;
    }
    pair = npair;
    tile = ntile;
  }
  cp_async_wait<0>();
  // fp16 holds |v| < 65504: a value at or past it marks the output invalid
  if constexpr (F16)
    if (!(vmax < 65504.0f) && status) atomicExch(status, kStatusF16Range);
}

__global__ void __launch_bounds__(THREADS, 2)
activation_kernel(const float *__restrict__ x, float *__restrict__ y, int rows, int C, int T,
                  int tiles_per_row, long long n_tiles, const float *__restrict__ log_alpha,
                  const float *__restrict__ log_beta, const float *__restrict__ f_up,
                  const float *__restrict__ f_dn, float eps) {
  activation_walk<false, K1_NX>(x, y, nullptr, rows, C, T, tiles_per_row, n_tiles, log_alpha,
                                log_beta, f_up, f_dn, eps);
}

// TW_ = 4: two 4-warp teams per CTA, two CTAs per SM; TW_ = 8: one 8-warp team
// per CTA, two CTAs per SM; TW_ = 16: one 16-warp team per CTA, one CTA per
// SM.  Each way 16 warps per SM.
template <int TW_, bool F16>
__global__ void __launch_bounds__(32 * TeamShape<TW_>::kCtaWarps, TW_ == 16 ? 1 : 2)
activation_tm_kernel(const float *__restrict__ x, float *__restrict__ hi, float *__restrict__ lo,
                     int rows, int C, int T, int tiles_per_row, long long n_tasks,
                     const float *__restrict__ log_alpha, const float *__restrict__ log_beta,
                     const float *__restrict__ f_up, const float *__restrict__ f_dn, float eps,
                     int *status) {
  activation_walk<true, TM_NX, TW_, F16>(x, hi, lo, rows, C, T, tiles_per_row, n_tasks,
                                         log_alpha, log_beta, f_up, f_dn, eps, status);
}

__global__ void sin_squared_kernel(const float *__restrict__ z, float *__restrict__ out,
                                   long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    out[i] = sin_squared(z[i]);
}

// CTAs resident at once for the activation kernel on the current device
// (computed once per device; a racing first call computes the same value).
int persistent_ctas() {
  constexpr int kMaxDev = 64;
  static std::atomic<int> cache[kMaxDev];
  int dev = 0;
  cudaGetDevice(&dev);
  const int slot = dev >= 0 && dev < kMaxDev ? dev : 0;
  int n = cache[slot].load(std::memory_order_relaxed);
  if (n == 0) {
    int sms = 148, per_sm = 2;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, activation_kernel, THREADS,
                                                      SMEM_BYTES) != cudaSuccess ||
        per_sm < 1)
      per_sm = 2;
    n = sms * per_sm;
    cache[slot].store(n, std::memory_order_relaxed);
  }
  return n;
}

template <int TW_>
int persistent_ctas_tm() {
  constexpr int kMaxDev = 64;
  static std::atomic<int> cache[kMaxDev];
  int dev = 0;
  cudaGetDevice(&dev);
  const int slot = dev >= 0 && dev < kMaxDev ? dev : 0;
  int n = cache[slot].load(std::memory_order_relaxed);
  if (n == 0) {
    int sms = 148, per_sm = 1;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &per_sm, activation_tm_kernel<TW_, false>, 32 * TeamShape<TW_>::kCtaWarps,
            tm_smem_bytes<TW_>()) != cudaSuccess ||
        per_sm < 1)
      per_sm = 1;
    n = sms * per_sm;
    cache[slot].store(n, std::memory_order_relaxed);
  }
  return n;
}

template <int TW_>
bv_status run_activation_tm(const float *x, float *hi, float *lo, long long rows, int C, int T,
                            const float *la, const float *lb, const float *fu, const float *fd,
                            float eps, cudaStream_t st, bool f16) {
  using S = TeamShape<TW_>;
  const int tiles = (T + TW - 1) / TW;
  const long long n_tasks = rows / S::kCh * tiles;  // (group, tile) tasks
  if (n_tasks <= 0) return BV_OK;
  BV_TRY(ensure_dynamic_smem(f16 ? (const void *)activation_tm_kernel<TW_, true>
                                 : (const void *)activation_tm_kernel<TW_, false>,
                             tm_smem_bytes<TW_>(), "activation_tm smem attribute"));
  const long long ctas = persistent_ctas_tm<TW_>();
  const long long need = (n_tasks + S::kTeams - 1) / S::kTeams;
  const long long grid = need < ctas ? need : ctas;
  {
    // algorithmic bytes: read x (4 B), write the hi and lo planes (8 B, or
    // 4 B in fp16)
    LaunchTimer tm(st, "activation_tm", 0.0, (f16 ? 8.0 : 12.0) * (double)rows * T);
    if (f16)
      activation_tm_kernel<TW_, true><<<(unsigned)grid, 32 * S::kCtaWarps, tm_smem_bytes<TW_>(),
                                        st>>>(x, hi, lo, (int)rows, C, T, tiles, n_tasks, la, lb,
                                              fu, fd, eps, device_status_ptr());
    else
      activation_tm_kernel<TW_, false><<<(unsigned)grid, 32 * S::kCtaWarps, tm_smem_bytes<TW_>(),
                                         st>>>(x, hi, lo, (int)rows, C, T, tiles, n_tasks, la, lb,
                                               fu, fd, eps, nullptr);
  }
  count_launch();
  return check_launch("activation_tm_kernel");
}

}  // namespace

bool activation_tm_supported(int C) { return C % TeamShape<4>::kCh == 0; }

bv_status launch_activation_tm(const float *x, float *hi, float *lo, int B, int C, int T,
                               const float *la, const float *lb, const float *fu, const float *fd,
                               float eps, cudaStream_t st, bool f16) {
  if (!activation_tm_supported(C))
    return fail(BV_ERR_UNSUPPORTED, "activation_tm: C = %d is not a multiple of %d", C,
                TeamShape<4>::kCh);
  if (((reinterpret_cast<uintptr_t>(hi) | reinterpret_cast<uintptr_t>(lo)) & 15u) != 0)
    return fail(BV_ERR_UNSUPPORTED, "activation_tm: planes not 16-byte aligned");
  const long long rows = (long long)B * C;
  if (rows > 0x7fffffffLL) return fail(BV_ERR_SHAPE, "activation_tm: too many rows");
  // the widest plane rows per time step the channels allow
  if (C % TeamShape<16>::kCh == 0)
    return run_activation_tm<16>(x, hi, lo, rows, C, T, la, lb, fu, fd, eps, st, f16);
  if (C % TeamShape<8>::kCh == 0)
    return run_activation_tm<8>(x, hi, lo, rows, C, T, la, lb, fu, fd, eps, st, f16);
  return run_activation_tm<4>(x, hi, lo, rows, C, T, la, lb, fu, fd, eps, st, f16);
}

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
  const int tiles = (T + TW - 1) / TW;
  const long long n_tiles = (rows + 1) / 2 * tiles;
  if (n_tiles <= 0) return BV_OK;
  if (rows > 0x7fffffffLL || (rows + 1) / 2 > 0x7fffffffLL / 2)
    return fail(BV_ERR_SHAPE, "activation: too many rows");
  BV_TRY(ensure_dynamic_smem((const void *)activation_kernel, SMEM_BYTES,
                             "activation smem attribute"));
  const long long ctas = persistent_ctas();
  const long long need = (n_tiles + WARPS - 1) / WARPS;
  const long long grid = need < ctas ? need : ctas;
  {
    LaunchTimer tm(st, "activation", 0.0, 8.0 * (double)rows * T);
    activation_kernel<<<(unsigned)grid, THREADS, SMEM_BYTES, st>>>(
        x, y, (int)rows, C, T, tiles, n_tiles, la, lb, fu, fd, eps);
  }
  count_launch();
  return check_launch("activation_kernel");
}

}  // namespace bv
