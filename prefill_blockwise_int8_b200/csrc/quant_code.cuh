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

// The same codes as quant_code for eight values, each as the bit pattern
// of the float code + 1.5 * 2^23.
//
// u = fl(x r + 1.5 * 2^23) (one fused multiply-add) lies in [2^23, 2^24),
// where floats are integers, so t = u - 1.5 * 2^23 is an integer near x r
// and u's low byte is t as a two's-complement int8: no float-to-int
// conversion is needed.  If the exact x r lies within 0.5 - 2^-13 of t
// (checked on fl(x r - t), one more fused multiply-add), t is also the
// integer nearest x / s, since |x / s - x r| stays below 2^-15 for
// |x / s| <= 128, hence t = rint(fl(x / s)); otherwise the code comes from
// the IEEE division.  The check is combined over the eight values, so the
// division path costs one rarely taken branch per eight codes.  No clamp:
// |x| <= absmax and s = fl(absmax / 127) keep |x / s| within
// 127 (1 + 3 * 2^-24) on both paths.  A zero block (s = 0, r = 0) gives
// code 0 for finite x.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ void quant_codes8(const float (&x)[8], float s,
                                             float r, uint32_t (&bits)[8]) {
  bool near_half = false;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float u = __fmaf_rn(x[e], r, kRoundMagic);
    const float t = __fsub_rn(u, kRoundMagic);
    near_half |= !(fabsf(__fmaf_rn(x[e], r, -t)) < 0.5f - 0x1p-13f);
    bits[e] = __float_as_uint(u);
  }
  if (near_half) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float u = __fmaf_rn(x[e], r, kRoundMagic);
      const float t = __fsub_rn(u, kRoundMagic);
      if (!(fabsf(__fmaf_rn(x[e], r, -t)) < 0.5f - 0x1p-13f))
        bits[e] = __float_as_uint(__fadd_rn(__fdiv_rn(x[e], s), kRoundMagic));
    }
  }
}

// Low bytes of four words (the code patterns above) -> one word, byte i
// from word i.
__device__ __forceinline__ uint32_t pack_low_bytes4(uint32_t a, uint32_t b,
                                                    uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040),
                     0x5410);
}

// The two fp16 halves of a 32-bit word as floats (exact).
__device__ __forceinline__ void half2_bits_to_float2(uint32_t w, float& lo,
                                                     float& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(w));
}

}  // namespace tilemix
