// Shared-memory operand layouts and small helpers of the fused attention
// kernels: tcgen05 descriptors of the K-major Q / K tiles and the MN-major V
// tile, the 128- and 64-byte swizzles the TMA loads write, and the exact
// INT8 -> fp16 conversion of the INT8 KV cache.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "ptx.cuh"

namespace tilemix {

// Routing paths of a 64-key half (bit set: some row takes that path).
constexpr uint32_t kKindF16 = 1, kKindI8 = 2;

// Lazy rescaling of the shared softmax state: the running row max only
// moves when a tile's max exceeds it by more than 2^8 (log2 units), so
// P <= 2^8 always fits fp16 and O is rescaled rarely.
constexpr float kRescaleThreshold = 8.0f;

// K-major fp16 operand stored as D/64 column chunks of [rows][128 B] with
// the 128-byte swizzle; `chunk_bytes` = rows * 128; ks = K-step of 16.
__device__ __forceinline__ uint64_t desc_k_f16(uint32_t base, int chunk_bytes,
                                               int ks) {
  const uint32_t addr = base + (ks >> 2) * chunk_bytes + (ks & 3) * 32;
  return smem_desc(addr, 16, 1024, kSwizzle128);
}

// Descriptor increment (16-byte units of the start address) from K-step 0
// to K-step ks of a K-major fp16 operand in one column chunk:
// desc_k_f16(b, c, ks) == desc_k_f16(b, c, 0) + k_step(ks) for ks < 4, while
// the start address stays below 2^18 bytes (all of shared memory), so the
// 14-bit field never carries.
__host__ __device__ constexpr uint64_t k_step(int ks) {
  return static_cast<uint64_t>(((ks & 3) * 32) >> 4);
}

// K-major int8 operand (rows x D bytes); ks = K-step of 32 bytes.
template <int D>
__device__ __forceinline__ uint64_t desc_k_i8(uint32_t base, int ks) {
  return smem_desc(base + ks * 32, 16, 8 * D,
                   D == 128 ? kSwizzle128 : kSwizzle64);
}

// MN-major fp16 V tile (keys x D) stored as D/64 chunks [keys][128 B] at
// `chunk_bytes` apart; ks = K-step of 16 keys.  LBO = chunk stride, SBO = 8
// keys.
__device__ __forceinline__ uint64_t desc_v(uint32_t base, int chunk_bytes,
                                           int ks) {
  return smem_desc(base + ks * 16 * 128, chunk_bytes, 1024, kSwizzle128);
}

// Byte offset inside a tile stored with the 128- (m = 7) or 64-byte (m = 3)
// swizzle: 16-byte unit bits [4:6] XOR row bits [7:9].
__device__ __forceinline__ uint32_t swz(uint32_t o, uint32_t m) {
  return o ^ (((o >> 7) & m) << 4);
}

// Four int8 (one word) -> two fp16 pairs, exactly: bias the bytes to
// unsigned, place each under the fp16 exponent of 1024 (0x64xx = 1024 +
// byte), subtract 1024 + 128.
__device__ __forceinline__ void i8x4_to_h2x2(uint32_t w, uint32_t& lo,
                                             uint32_t& hi) {
  const uint32_t x = w ^ 0x80808080u;
  const __half2 bias = __float2half2_rn(1152.0f);
  uint32_t a = __byte_perm(x, 0x64646464u, 0x4140);
  uint32_t b = __byte_perm(x, 0x64646464u, 0x4342);
  __half2 ha = __hsub2(*reinterpret_cast<__half2*>(&a), bias);
  __half2 hb = __hsub2(*reinterpret_cast<__half2*>(&b), bias);
  lo = *reinterpret_cast<uint32_t*>(&ha);
  hi = *reinterpret_cast<uint32_t*>(&hb);
}

// One key row of an INT8 tile (D bytes at row rr of `src`, swizzled with
// mask sm, 0 = plain rows) -> the fp16 K-major / V layout: D/64 chunks of
// [rows][128 B] with the 128-byte swizzle, CHUNK bytes apart.  With SCALE,
// each value is multiplied by s2 (rounded once to fp16).  The whole row is
// read before any store, so the fp16 row may overlap the INT8 row it came
// from.
template <int D, bool SCALE, int CHUNK>
__device__ __forceinline__ void convert_row(const uint8_t* src, uint32_t sm,
                                            uint8_t* dst, int rr,
                                            __half2 s2) {
  uint4 in[D / 16];
#pragma unroll
  for (int u = 0; u < D / 16; ++u)
    in[u] = *reinterpret_cast<const uint4*>(src + swz(rr * D + u * 16, sm));
#pragma unroll
  for (int u = 0; u < D / 16; ++u) {
    const uint32_t w[4] = {in[u].x, in[u].y, in[u].z, in[u].w};
    uint32_t h[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) i8x4_to_h2x2(w[i], h[2 * i], h[2 * i + 1]);
    if (SCALE) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        __half2 v = __hmul2(*reinterpret_cast<__half2*>(&h[i]), s2);
        h[i] = *reinterpret_cast<uint32_t*>(&v);
      }
    }
    // dims 16u .. 16u+15 -> chunk (16u) / 64, 16-byte units 2u, 2u+1 of it
    const int c = (16 * u) / 64;
    const int uo = (2 * u) % 8;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const uint32_t o = c * CHUNK + rr * 128 + (uo + e) * 16;
      *reinterpret_cast<uint4*>(dst + swz(o, 7)) =
          make_uint4(h[4 * e], h[4 * e + 1], h[4 * e + 2], h[4 * e + 3]);
    }
  }
}

}  // namespace tilemix
