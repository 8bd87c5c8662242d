// One INT8 code of the blockwise symmetric quantiser, shared by the
// quantise-once kernel and the attention kernel's on-chip mode so that both
// produce identical codes: code = clamp(rint(fl(x / s)), -127, 127) with an
// IEEE fp32 division, s = fl(absmax / 127).
#pragma once

#include <cuda_runtime.h>

namespace tilemix {

// code = rint(fl(x / s)) without a division per element: y = x * fl(1/s)
// lies within a few ulp of fl(x / s) (|y| <= 128, so within 2^-15), hence
// both round to the same integer unless y is within that distance of a
// half-integer; those rare elements take the IEEE division.
__device__ __forceinline__ int quant_code(float x, float s, float r) {
  const float y = x * r;
  const float t = rintf(y);
  const float frac = fabsf(y - t);  // in [0, 0.5] (+ rounding)
  int q;
  if (frac < 0.5f - 0x1p-13f) {
    q = static_cast<int>(t);
  } else {
    q = __float2int_rn(__fdiv_rn(x, s));
  }
  return max(-127, min(127, q));
}


}  // namespace tilemix
