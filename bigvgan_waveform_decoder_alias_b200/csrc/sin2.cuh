// sin^2(z) for the SnakeBeta term, in FP32 on the FMA pipe.
//
// sin^2 has period pi, so z is reduced to r = z - k pi with k = rint(z / pi)
// and |r| <= pi/2 (Cody & Waite's additive reduction, "Software Manual for
// the Elementary Functions", 1980): pi is split as C1 + C2 + C3 where C1 =
// 3.140625 has 8 significant bits, so k C1 is exact for |k| < 2^16, and C2,
// C3 are the next two float parts of pi; the last two products go through
// FMA.  Then sin(r) = r (1 - r^2/3! + r^4/5! - ... - r^12/13!) -- the Taylor
// series of sin cut after the r^13 term, whose remainder on |r| <= pi/2 is
// below (pi/2)^15 / 15! = 6.6e-10 -- and sin^2 = sin(r)^2.
// For |z| > 65536 (never met by a decoder's signals) it falls back to sinf.
#pragma once

namespace bv {

namespace sin2c {
constexpr float kInvPi = 0.31830987334251404f;      // float(1/pi)
constexpr float kC1 = 3.140625f;                     // 201/64
constexpr float kC2 = 0.0009676535846665502f;        // float(pi - C1)
constexpr float kC3 = 5.126688136514179e-12f;        // float(pi - C1 - C2)
constexpr float kT1 = -0.1666666716337204f;          // -1/3!
constexpr float kT2 = 0.008333333767950535f;         //  1/5!
constexpr float kT3 = -0.00019841270113829523f;      // -1/7!
constexpr float kT4 = 2.7557318844628753e-06f;       //  1/9!
constexpr float kT5 = -2.5052107943679403e-08f;      // -1/11!
constexpr float kT6 = 1.6059044372074283e-10f;       //  1/13!
constexpr float kFastLimit = 65536.0f;
}  // namespace sin2c

// sin(pi f) for |f| <= 1/2 as f P(f^2), P of degree 4: coefficients of a
// near-minimax fit of sin(pi f) / f in s = f^2 on [0, 1/4] (least squares on
// Chebyshev nodes, reweighted by Lawson's iteration towards the minimax
// error), rounded to float.  Approximation error 3.4e-9 before and 4.9e-8
// after the rounding; evaluated by Horner's rule in float, within 2.5e-7.
namespace sin2p {
constexpr float kInvPi = 0.31830987334251404f;  // float(1/pi)
__host__ __device__ constexpr float coef(int j) {
  return j == 0   ? 3.141592502593994f
         : j == 1 ? -5.1677069664001465f
         : j == 2 ? 2.5500314235687256f
         : j == 3 ? -0.5980451703071594f
                  : 0.0772201344370842f;
}
}  // namespace sin2p

__device__ __forceinline__ float sin_squared_reduced(float z) {
  using namespace sin2c;
  const float k = rintf(z * kInvPi);
  float r = fmaf(-k, kC1, z);
  r = fmaf(-k, kC2, r);
  r = fmaf(-k, kC3, r);
  const float r2 = r * r;
  float p = fmaf(r2, kT6, kT5);
  p = fmaf(r2, p, kT4);
  p = fmaf(r2, p, kT3);
  p = fmaf(r2, p, kT2);
  p = fmaf(r2, p, kT1);
  p = fmaf(r2, p, 1.0f);
  const float s = r * p;
  return s * s;
}

__device__ __forceinline__ float sin_squared(float z) {
  if (fabsf(z) <= sin2c::kFastLimit) return sin_squared_reduced(z);
  const float s = sinf(z);
  return s * s;
}

}  // namespace bv
