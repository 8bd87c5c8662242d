// Blockwise symmetric INT8 quantiser ("quantize-once") for sm_100a.
//
// Method: TileMix (arXiv 2608.17336), paperlayer summary section 3
// Preliminaries (blockwise quantization, INT8 tensor cores with INT32
// accumulation) and appendix C Quantization Configuration (Q and K
// quantised blockwise and symmetrically once per attention call).
// Per (sequence, head, block of tokens): scale = absmax / 127 (IEEE fp32
// division), code = clamp(round_half_even(x / scale), -127, 127).
//
// HBM-bound: one CTA copies one block (up to 64 KB of fp16) once into
// shared memory with 16-byte asynchronous copies (cp.async: few registers,
// so six CTAs per SM keep their loads in flight together), reduces the
// absmax, and writes the codes with 8-byte stores.  One launch can serve two tensors (Q and K): grid.y
// runs over the heads of the first, then of the second, so both share one
// grid and the short tail of a single launch is paid once.  Rows of a block are strided by heads * d in memory,
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

// 16-byte global -> shared copy that bypasses L1 and registers; completes
// for the issuing thread at cp_async_wait_all().
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
}

// One tensor of a launch: x [T, heads, d] -> x8, scale [heads, batch, nblk].
struct QuantJob {
  const __half* x;
  int8_t* x8;
  float* scale;
  int heads, block, nblk;
};

// VPT 16-byte vectors (8 halves) per thread; VPR vectors per row (d / 8),
// 0 = taken from vpr_rt at run time.  Heads [0, j0.heads) of grid.y are
// j0's, the rest j1's (j1.heads = 0 for a single tensor).
template <int VPT, int VPR>
__global__ void __launch_bounds__(kQThreads)
    quantize_kernel(const QuantJob j0, const QuantJob j1,
                    const int32_t* __restrict__ cu_seqlens, int batch,
                    int max_seqlen, int total_tokens, int vpr_rt,
                    int32_t* status) {
  const int vpr = VPR > 0 ? VPR : vpr_rt;
  const int d = vpr * 8;
  const bool second = static_cast<int>(blockIdx.y) >= j0.heads;
  const __half* __restrict__ x = second ? j1.x : j0.x;
  int8_t* __restrict__ x8 = second ? j1.x8 : j0.x8;
  float* __restrict__ scale = second ? j1.scale : j0.scale;
  const int heads = second ? j1.heads : j0.heads;
  const int block = second ? j1.block : j0.block;
  const int nblk = second ? j1.nblk : j0.nblk;
  const int t = blockIdx.x;
  const int h = second ? blockIdx.y - j0.heads : blockIdx.y;
  const int b = blockIdx.z;
  if (t >= nblk) return;
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
  // row's VPR vectors are one coalesced read.  A thread only reads back the
  // vectors it copied itself, so its own wait orders them.
  extern __shared__ uint4 stage[];
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const int idx = threadIdx.x + k * kQThreads;
    if (idx < nv) {
      const int r = idx / vpr;
      const int c = idx % vpr;
      cp_async16(&stage[idx],
                 reinterpret_cast<const uint4*>(base + r * row_stride) + c);
    }
  }
  cp_async_wait_all();
  __half2 amax2 = __float2half2_rn(0.0f);
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const int idx = threadIdx.x + k * kQThreads;
    if (idx < nv) {
      const uint4 vk = stage[idx];
      const __half2* hv = reinterpret_cast<const __half2*>(&vk);
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
      const uint4 vk = stage[idx];
      const uint32_t w4[4] = {vk.x, vk.y, vk.z, vk.w};
      float f[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) half2_bits_to_float2(w4[e], f[2 * e], f[2 * e + 1]);
      uint32_t cb[8];
      quant_codes8(f, s, rcp, cb);
      *reinterpret_cast<uint2*>(qbase + r * row_stride + c * 8) =
          make_uint2(pack_low_bytes4(cb[0], cb[1], cb[2], cb[3]),
                     pack_low_bytes4(cb[4], cb[5], cb[6], cb[7]));
    }
  }
}

template <int VPR>
cudaError_t launch_vpr(dim3 grid, int vecs, cudaStream_t stream,
                       const QuantJob& j0, const QuantJob& j1,
                       const int32_t* cu_seqlens, int batch, int max_seqlen,
                       int total_tokens, int vpr_rt, int32_t* status) {
  const int vpt = (vecs + kQThreads - 1) / kQThreads;
  const int smem = vecs * 16;  // one block of fp16, <= 64 KB
  auto go = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(
        kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kQThreads, smem, stream>>>(j0, j1, cu_seqlens, batch,
                                            max_seqlen, total_tokens, vpr_rt,
                                            status);
    return cudaGetLastError();
  };
  if (vpt <= 2) return go(quantize_kernel<2, VPR>);
  if (vpt <= 4) return go(quantize_kernel<4, VPR>);
  if (vpt <= 8) return go(quantize_kernel<8, VPR>);
  if (vpt <= 16) return go(quantize_kernel<16, VPR>);
  return cudaErrorInvalidValue;
}

cudaError_t launch_jobs(const QuantJob& j0, const QuantJob& j1,
                        const int32_t* cu_seqlens, int batch, int max_seqlen,
                        int total_tokens, int head_dim, int32_t* status,
                        cudaStream_t stream) {
  dim3 grid(max(j0.nblk, j1.nblk), j0.heads + j1.heads, batch);
  const int vecs = max(j0.block, j1.block) * head_dim / 8;
  const int vpr = head_dim / 8;
  if (head_dim == 128)
    return launch_vpr<16>(grid, vecs, stream, j0, j1, cu_seqlens, batch,
                          max_seqlen, total_tokens, vpr, status);
  if (head_dim == 64)
    return launch_vpr<8>(grid, vecs, stream, j0, j1, cu_seqlens, batch,
                         max_seqlen, total_tokens, vpr, status);
  return launch_vpr<0>(grid, vecs, stream, j0, j1, cu_seqlens, batch,
                       max_seqlen, total_tokens, vpr, status);
}

}  // namespace

cudaError_t launch_quantize_blockwise(const void* x, const int32_t* cu_seqlens,
                                      int batch, int max_seqlen,
                                      int total_tokens, int heads,
                                      int head_dim, int block, int8_t* x8,
                                      float* scale, int32_t* status,
                                      cudaStream_t stream) {
  const QuantJob j0{static_cast<const __half*>(x), x8, scale, heads, block,
                    (max_seqlen + block - 1) / block};
  const QuantJob j1{nullptr, nullptr, nullptr, 0, 1, 0};
  return launch_jobs(j0, j1, cu_seqlens, batch, max_seqlen, total_tokens,
                     head_dim, status, stream);
}

cudaError_t launch_quantize_blockwise_qk(
    const void* q, const void* k, const int32_t* cu_seqlens, int batch,
    int max_seqlen, int total_tokens, int hq, int hkv, int head_dim,
    int block_q, int block_k, int8_t* q8, float* q_scale, int8_t* k8,
    float* k_scale, int32_t* status, cudaStream_t stream) {
  const QuantJob jq{static_cast<const __half*>(q), q8, q_scale, hq, block_q,
                    (max_seqlen + block_q - 1) / block_q};
  const QuantJob jk{static_cast<const __half*>(k), k8, k_scale, hkv, block_k,
                    (max_seqlen + block_k - 1) / block_k};
  return launch_jobs(jq, jk, cu_seqlens, batch, max_seqlen, total_tokens,
                     head_dim, status, stream);
}

}  // namespace tilemix
