// sin^2 for the SnakeBeta term.
#pragma once

namespace bv {

__device__ __forceinline__ float sin_squared(float z) {
  const float s = sinf(z);
  return s * s;
}

}  // namespace bv
