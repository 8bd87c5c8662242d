// Blockwise symmetric INT8 quantiser ("quantize-once") for sm_100a.
//
// Method: TileMix (arXiv 2608.17336), paperlayer summary section 3
// Preliminaries (blockwise quantization, INT8 tensor cores with INT32
// accumulation) and appendix C Quantization Configuration (Q and K
// quantised blockwise and symmetrically once per attention call).
// Per (sequence, head, block of tokens): scale = absmax / 127 (IEEE fp32
// division), code = clamp(round_half_even(x / scale), -127, 127).
//
// HBM-bound: one CTA reads one block (up to 32 KB of fp16) once into
// registers with 16-byte loads, reduces the absmax, and writes the codes
// with 8-byte stores.  Rows of a block are strided by heads * d in memory,
// each row contiguous.  The per-element IEEE division is replaced by a
// multiply with the reciprocal wherever that provably gives the same code,
// and the integer code is read off a float's bit pattern (no conversion
// instruction).
#include <cuda_fp16.h>
#include <stdint.h>

#include "internal.h"
#include "quant_code.cuh"

namespace tilemix {
namespace {

constexpr int kQThreads = 256;

// VPT 16-byte vectors (8 halves) per thread; VPR vectors per row (d / 8),
// 0 = taken from vpr_rt at run time.
template <int VPT, int VPR>
__global__ void __launch_bounds__(kQThreads)
    quantize_kernel(const __half* __restrict__ x,
                    const int32_t* __restrict__ cu_seqlens, int batch,
                    int max_seqlen, int total_tokens, int heads, int block,
                    int nblk, int vpr_rt, int8_t* __restrict__ x8,
                    float* __restrict__ scale, int32_t* status) {
  const int vpr = VPR > 0 ? VPR : vpr_rt;
  const int d = vpr * 8;
  const int t = blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int start = cu_seqlens[b];
  const int len = cu_seqlens[b + 1] - start;
  if (start < 0 || len < 0 || len > max_seqlen || start + len > total_tokens) {
    if (threadIdx.x == 0) report_status(status, kStatusBadSeqlens);
    return;
  }
  float* s_out = scale + (static_cast<size_t>(h) * batch + b) * nblk + t;
  const int r0 = t * block;
  if (r0 >= len) {
    if (threadIdx.x == 0) *s_out = 0.0f;
    return;
  }
  const int rows = min(block, len - r0);
  const int nv = rows * vpr;
  const size_t row_stride = static_cast<size_t>(heads) * d;
  const __half* base = x + (static_cast<size_t>(start + r0) * heads + h) * d;

  // Consecutive threads take consecutive 16-byte vectors of a row, so each
  // row's VPR vectors are one coalesced read.
  uint4 v[VPT];
  __half2 amax2 = __float2half2_rn(0.0f);
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const int idx = threadIdx.x + k * kQThreads;
    if (idx < nv) {
      const int r = idx / vpr;
      const int c = idx % vpr;
      v[k] = __ldg(reinterpret_cast<const uint4*>(base + r * row_stride) + c);
      const __half2* hv = reinterpret_cast<const __half2*>(&v[k]);
#pragma unroll
      for (int e = 0; e < 4; ++e) amax2 = __hmax2(amax2, __habs2(hv[e]));
    }
  }
  float amax = fmaxf(__low2float(amax2), __high2float(amax2));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  __shared__ float warp_max[kQThreads / 32];
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = warp_max[0];
#pragma unroll
  for (int w = 1; w < kQThreads / 32; ++w) amax = fmaxf(amax, warp_max[w]);

  const float s = __fdiv_rn(amax, 127.0f);
  const float rcp = amax != 0.0f ? __frcp_rn(s) : 0.0f;
  if (threadIdx.x == 0) *s_out = s;
  int8_t* qbase = x8 + (static_cast<size_t>(start + r0) * heads + h) * d;
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const int idx = threadIdx.x + k * kQThreads;
    if (idx < nv) {
      const int r = idx / vpr;
      const int c = idx % vpr;
      const uint32_t w4[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
      float f[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) half2_bits_to_float2(w4[e], f[2 * e], f[2 * e + 1]);
      uint32_t cb[8];
      quant_codes8(f, s, rcp, cb);
      // low bytes of four patterns -> one word
      auto pack4 = [](uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
        return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040),
                           0x5410);
      };
      *reinterpret_cast<uint2*>(qbase + r * row_stride + c * 8) =
          make_uint2(pack4(cb[0], cb[1], cb[2], cb[3]),
                     pack4(cb[4], cb[5], cb[6], cb[7]));
    }
  }
}

template <int VPR>
cudaError_t launch_vpr(dim3 grid, int vecs, cudaStream_t stream,
                       const __half* x, const int32_t* cu_seqlens, int batch,
                       int max_seqlen, int total_tokens, int heads, int block,
                       int nblk, int vpr_rt, int8_t* x8, float* scale,
                       int32_t* status) {
  const int vpt = (vecs + kQThreads - 1) / kQThreads;
#define TILEMIX_QLAUNCH(N)                                                  \
  quantize_kernel<N, VPR><<<grid, kQThreads, 0, stream>>>(                  \
      x, cu_seqlens, batch, max_seqlen, total_tokens, heads, block, nblk,   \
      vpr_rt, x8, scale, status)
  if (vpt <= 2) TILEMIX_QLAUNCH(2);
  else if (vpt <= 4) TILEMIX_QLAUNCH(4);
  else if (vpt <= 8) TILEMIX_QLAUNCH(8);
  else if (vpt <= 16) TILEMIX_QLAUNCH(16);
  else return cudaErrorInvalidValue;
#undef TILEMIX_QLAUNCH
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_blockwise(const void* x, const int32_t* cu_seqlens,
                                      int batch, int max_seqlen,
                                      int total_tokens, int heads,
                                      int head_dim, int block, int8_t* x8,
                                      float* scale, int32_t* status,
                                      cudaStream_t stream) {
  const int nblk = (max_seqlen + block - 1) / block;
  dim3 grid(nblk, heads, batch);
  const __half* xh = static_cast<const __half*>(x);
  const int vecs = block * head_dim / 8;
  const int vpr = head_dim / 8;
  if (head_dim == 128)
    return launch_vpr<16>(grid, vecs, stream, xh, cu_seqlens, batch,
                          max_seqlen, total_tokens, heads, block, nblk, vpr,
                          x8, scale, status);
  if (head_dim == 64)
    return launch_vpr<8>(grid, vecs, stream, xh, cu_seqlens, batch,
                         max_seqlen, total_tokens, heads, block, nblk, vpr, x8,
                         scale, status);
  return launch_vpr<0>(grid, vecs, stream, xh, cu_seqlens, batch, max_seqlen,
                       total_tokens, heads, block, nblk, vpr, x8, scale,
                       status);
}

}  // namespace tilemix
