// Routing-word packer for sm_100a.
//
// Method: TileMix (arXiv 2608.17336), paperlayer summary section 3
// Preliminaries (routing groups adjacent key tiles into packed 64-bit masks;
// bit floor(n/g) selects INT8 or FP16 for key tile n; legality masks act
// independently) and section 4 (the routing map is indexed by KV head,
// query-tile row and key-tile group; O(H_k T_m) words).
//
// One thread per word: read the row's 64 route bytes with four 16-byte
// loads, set bit j for every nonzero byte, then clear the bits of groups
// past the last one that holds a legal (causal, in-sequence) key.
#include <stdint.h>

#include "internal.h"

namespace tilemix {
namespace {

__global__ void __launch_bounds__(256)
    pack_mask_kernel(const uint8_t* __restrict__ route,
                     const int32_t* __restrict__ cu_seqlens, int batch,
                     int max_seqlen, int hkv, int tm, int block_m, int block_n,
                     int group, uint64_t* __restrict__ mask, int32_t* status) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x +
                        threadIdx.x;
  const long long total = static_cast<long long>(batch) * hkv * tm;
  if (idx >= total) return;
  const int m = static_cast<int>(idx % tm);
  const int b = static_cast<int>(idx / (static_cast<long long>(hkv) * tm));
  const int len = cu_seqlens[b + 1] - cu_seqlens[b];
  if (len < 0 || len > max_seqlen) {
    report_status(status, kStatusBadSeqlens);
    mask[idx] = 0;
    return;
  }
  uint64_t word = 0;
  if (static_cast<long long>(m) * block_m < len) {
    const int last_row = min((m + 1) * block_m, len) - 1;
    const int g_last = (last_row / block_n) / group;  // <= 63 (host check)
    const uint4* src = reinterpret_cast<const uint4*>(route + idx * 64);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint4 q = __ldg(src + v);
      const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int byte = 0; byte < 4; ++byte)
          if ((w4[k] >> (8 * byte)) & 0xffu)
            word |= 1ull << (v * 16 + k * 4 + byte);
    }
    if (g_last < 63) word &= (2ull << g_last) - 1ull;
  }
  mask[idx] = word;
}

}  // namespace

cudaError_t launch_pack_mask(const uint8_t* route, const int32_t* cu_seqlens,
                             int batch, int max_seqlen, int hkv, int block_m,
                             int block_n, int group, uint64_t* mask,
                             int32_t* status, cudaStream_t stream) {
  const int tm = (max_seqlen + block_m - 1) / block_m;
  const long long total = static_cast<long long>(batch) * hkv * tm;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  pack_mask_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      route, cu_seqlens, batch, max_seqlen, hkv, tm, block_m, block_n, group,
      mask, status);
  return cudaGetLastError();
}

}  // namespace tilemix
