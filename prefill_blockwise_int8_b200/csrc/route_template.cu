// Static routing templates for sm_100a: route bytes of a named layout at a
// given INT8 coverage.
//
// Method: TileMix (arXiv 2608.17336), paperlayer summary appendix B
// Precision Layouts (All INT8 / All FP16 references and the Band, Global,
// Row-Random, Aligned Sparse, BigBird and SpTrans templates; coverage = INT8
// share of legal tile groups) and Limitations (static templates, any policy
// consumable by the kernel).  The pages name the layouts only; the priority
// rules are this library's readings (stated with the C declaration).
//
// One thread per query-tile row (b, hk, m): priorities and hashes of its
// <= 64 legal groups, rank of each group by (priority, hash, -j), FP16 for
// the top G - k_int8 ranks.
#include <stdint.h>

#include "internal.h"

namespace tilemix {
namespace {

__device__ __forceinline__ uint64_t splitmix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint32_t priority(int layout, int j, int d) {
  switch (layout) {
    case kLayoutBand: return static_cast<uint32_t>(63 - d);
    case kLayoutGlobal: return static_cast<uint32_t>(63 - j);
    case kLayoutAligned: return (j % 4 == 0) ? 1u : 0u;
    case kLayoutBigBird: return (j == 0 || d <= 1) ? 1u : 0u;
    case kLayoutSpTrans: return d <= 1 ? 2u : ((j % 4 == 3) ? 1u : 0u);
    default: return 0u;  // row-random
  }
}

__global__ void __launch_bounds__(128)
    route_template_kernel(int layout, int permille, uint64_t seed,
                          const int32_t* __restrict__ cu_seqlens, int batch,
                          int max_seqlen, int hkv, int tm, int block_m,
                          int block_n, int group, uint8_t* __restrict__ route,
                          int32_t* status) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x +
                        threadIdx.x;
  const long long total = static_cast<long long>(batch) * hkv * tm;
  if (idx >= total) return;
  const int m = static_cast<int>(idx % tm);
  const int b = static_cast<int>(idx / (static_cast<long long>(hkv) * tm));
  uint4* out = reinterpret_cast<uint4*>(route + idx * 64);
  const int len = cu_seqlens[b + 1] - cu_seqlens[b];
  int G = 0;
  if (len < 0 || len > max_seqlen) {
    report_status(status, kStatusBadSeqlens);
  } else if (static_cast<long long>(m) * block_m < len) {
    const int last_row = min((m + 1) * block_m, len) - 1;
    G = (last_row / block_n) / group + 1;  // <= 64 (host check)
  }
  uint64_t key[64];
#pragma unroll 1
  for (int j = 0; j < G; ++j) {
    const uint64_t c = static_cast<uint64_t>(idx) * 64ull + j;
    const uint64_t h =
        splitmix64(seed + (c + 1ull) * 0x9E3779B97F4A7C15ull) >> 32;
    key[j] = (static_cast<uint64_t>(priority(layout, j, G - 1 - j)) << 32) | h;
  }
  int k_int8 = (permille * G + 500) / 1000;
  if (layout == kLayoutAllFp16) k_int8 = 0;
  if (layout == kLayoutAllInt8) k_int8 = G;
  const int k_fp16 = G - k_int8;
  uint32_t bytes[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) bytes[i] = 0u;
#pragma unroll 1
  for (int j = 0; j < G; ++j) {
    int rank = 0;  // groups ahead of j: larger key, or equal key and smaller index
    for (int i = 0; i < G; ++i)
      rank += (key[i] > key[j] || (key[i] == key[j] && i < j)) ? 1 : 0;
    if (rank >= k_fp16) bytes[j >> 2] |= 1u << (8 * (j & 3));
  }
#pragma unroll
  for (int v = 0; v < 4; ++v)
    out[v] = make_uint4(bytes[4 * v], bytes[4 * v + 1], bytes[4 * v + 2],
                        bytes[4 * v + 3]);
}

}  // namespace

cudaError_t launch_route_template(int layout, int permille, uint64_t seed,
                                  const int32_t* cu_seqlens, int batch,
                                  int max_seqlen, int hkv, int block_m,
                                  int block_n, int group, uint8_t* route,
                                  int32_t* status, cudaStream_t stream) {
  const int tm = (max_seqlen + block_m - 1) / block_m;
  const long long total = static_cast<long long>(batch) * hkv * tm;
  if (total == 0) return cudaSuccess;
  const int threads = 128;
  const long long blocks = (total + threads - 1) / threads;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  route_template_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      layout, permille, seed, cu_seqlens, batch, max_seqlen, hkv, tm, block_m,
      block_n, group, route, status);
  return cudaGetLastError();
}

}  // namespace tilemix
