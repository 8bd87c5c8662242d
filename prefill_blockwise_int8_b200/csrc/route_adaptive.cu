// Adaptive routing from exact block logit sums, for sm_100a.
//
// Method: TileMix (arXiv 2608.17336), paperlayer summary Limitations (the
// kernel interface consumes static or adaptive routing policies) and
// appendix G.5 (routing that keeps high-mass attention blocks in FP16).  The
// statistic is this library's reading (stated with the C declaration): the
// sum of all raw logits between a query-tile row and a key group, computed
// exactly as (sum of the row's queries) . (sum of the group's keys) with
// fp16 values scaled to exact integers, so the result and the ranking do not
// depend on the order of any sum.
//
// Pass 1 (sums_kernel): one CTA per (query tile, or run of key groups of
// about 256 keys; KV head; sequence); each thread reads 16-byte chunks of
// rows (coalesced across the CTA) and keeps eight exact channel sums
// (rescaled doubles for runs, then int64); the CTA adds the slices' totals
// through shared memory.  Q and K are each read once.
// Pass 2 (rank_kernel): one CTA per (sequence, KV head, query-tile row);
// thread j forms the dot product of the row's sums with group j's in 24-bit
// limbs, ranks group j, writes its route byte, and warp ballots give the
// packed routing word.
#include <cuda_fp16.h>
#include <stdint.h>

#include "internal.h"
#include "tilemix.h"

namespace tilemix {
namespace {

constexpr int kGroups = 64;
constexpr int kSumThreads = 128;

// Exact sums of fp16 values in doubles, without a conversion instruction.
//
// Placing the 15 magnitude bits of an fp16 value (5 exponent, 10 mantissa)
// at the top of a double's exponent and mantissa fields, with the sign bit
// moved along, gives exactly the value times 2^-1008: an exponent field e
// reads as 2^(e - 1023) (1 + m / 1024) = 2^-1008 * 2^(e - 15) (1 + m / 1024),
// and e = 0 reads as the subnormal 2^-1022 m / 2^52 * 2^42 = 2^-1008 m 2^-24.
// Every such value is a multiple of 2^-1032 below 2^-992 in magnitude, so a
// double sum of at most 2^13 of them is a multiple of 2^-1032 below 2^-979:
// it needs at most 53 significant bits and every addition is exact
// (subnormal doubles are kept; nothing here flushes them).  Runs of at most
// kExactRun rows are summed so and moved, times 2^1032 (exact), into int64
// totals of value * 2^24.  (An Inf or NaN input gives an unspecified
// ranking.)
constexpr int kExactRun = 4096;

__device__ __forceinline__ double scaled_lo(uint32_t w) {
  const uint32_t hi = ((w & 0x7fffu) << 10) | ((w << 16) & 0x80000000u);
  return __hiloint2double(static_cast<int>(hi), 0);
}

__device__ __forceinline__ double scaled_hi(uint32_t w) {
  const uint32_t hi = ((w >> 6) & 0x01fffc00u) | (w & 0x80000000u);
  return __hiloint2double(static_cast<int>(hi), 0);
}

__device__ __forceinline__ void add_chunk(double (&a)[8], uint4 w) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a[2 * i] += scaled_lo(u[i]);
    a[2 * i + 1] += scaled_hi(u[i]);
  }
}

// Running exact sums of one thread's eight channels: doubles for runs of at
// most kExactRun rows, then int64 totals of value * 2^24.  The totals live
// in shared memory (t[e * kSumThreads], one column per thread): they change
// once per run, and the registers they would take go to loads in flight.
struct ExactSums {
  double a[8];
  int64_t* t;
  int run;

  __device__ __forceinline__ void clear() {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      a[e] = 0.0;
      t[e * kSumThreads] = 0;
    }
    run = 0;
  }
  __device__ __forceinline__ void settle() {
    // 2^1032 in two exact power-of-two steps (2^1032 is not a double)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      t[e * kSumThreads] += __double2ll_rn(a[e] * 0x1p1000 * 0x1p32);
      a[e] = 0.0;
    }
    run = 0;
  }
  // rows first, first + step, ... < last of a [rows, stride] fp16 matrix,
  // 16-byte chunk at `base`.  Eight rows at a time: their loads are issued
  // together, so each thread keeps 128 bytes in flight.
  __device__ __forceinline__ void add_rows(const uint16_t* __restrict__ base,
                                           size_t stride, int first, int last,
                                           int step) {
    constexpr int kBatch = 8;  // kExactRun is a multiple of it
    const uint16_t* p = base + static_cast<size_t>(first) * stride;
    const size_t dp = static_cast<size_t>(step) * stride;
    int i = first;
    for (; i + (kBatch - 1) * step < last; i += kBatch * step) {
      uint4 w[kBatch];
#pragma unroll
      for (int r = 0; r < kBatch; ++r)
        w[r] = __ldg(reinterpret_cast<const uint4*>(p + r * dp));
      p += kBatch * dp;
      if (run + kBatch > kExactRun) settle();
#pragma unroll
      for (int r = 0; r < kBatch; ++r) add_chunk(a, w[r]);
      run += kBatch;
    }
    for (; i < last; i += step, p += dp) {
      if (run == kExactRun) settle();
      add_chunk(a, __ldg(reinterpret_cast<const uint4*>(p)));
      ++run;
    }
  }
};

// The CTA's slices hold totals for the same channels; add them in order.
__device__ __forceinline__ void reduce_slices(const ExactSums& s,
                                              int64_t* part_s, int rs, int cc,
                                              int slices, int d,
                                              int64_t* __restrict__ out) {
  if (rs < slices) {
#pragma unroll
    for (int e = 0; e < 8; ++e) part_s[rs * d + cc * 8 + e] = s.t[e * kSumThreads];
  }
  __syncthreads();
  for (int c = threadIdx.x; c < d; c += kSumThreads) {
    int64_t total = 0;
    for (int r = 0; r < slices; ++r) total += part_s[r * d + c];
    out[c] = total;
  }
  __syncthreads();
}

// blockIdx.x < tm: query tile u (its rows over the KV head's query heads);
// otherwise key groups gpc * (x - tm) .. + gpc - 1 (groups past 63 skipped).
__global__ void __launch_bounds__(kSumThreads)
    sums_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                const int32_t* __restrict__ cu_seqlens,
                const int32_t* __restrict__ head_map, int max_seqlen,
                int total_tokens, int hq, int hkv, int d, int tm, int block_m,
                int keys_per_group, int gpc, int64_t* __restrict__ sq,
                int64_t* __restrict__ sk, int32_t* status) {
  // per-slice channel totals: slices * d = 8 * kSumThreads entries
  __shared__ int64_t part_s[8 * kSumThreads];
  const int u = blockIdx.x;
  const int hk = blockIdx.y;
  const int b = blockIdx.z;
  const int chunks = d >> 3;
  const int slices = kSumThreads / chunks;
  const int cc = threadIdx.x % chunks;
  const int rs = threadIdx.x / chunks;
  const int start = cu_seqlens[b];
  const int len = cu_seqlens[b + 1] - start;
  const bool valid = start >= 0 && len >= 0 && len <= max_seqlen &&
                     start + len <= total_tokens;
  if (!valid && threadIdx.x == 0 && u == 0 && hk == 0)
    report_status(status, kStatusBadSeqlens);
  const bool active = valid && rs < slices;
  __shared__ int64_t totals_s[8 * kSumThreads];
  ExactSums s;
  s.t = totals_s + threadIdx.x;
  s.clear();
  if (u < tm) {
    if (active) {
      const int r0 = u * block_m + rs, r1 = min((u + 1) * block_m, len);
      const size_t stride = static_cast<size_t>(hq) * d;
      const uint16_t* base = q + static_cast<size_t>(start) * stride + cc * 8;
      if (head_map) {
        for (int h = 0; h < hq; ++h) {
          const int hm = head_map[h];
          if (hm < 0 || hm >= hkv) {
            if (threadIdx.x == 0) report_status(status, kStatusBadSeqlens);
          } else if (hm == hk) {
            s.add_rows(base + static_cast<size_t>(h) * d, stride, r0, r1, slices);
          }
        }
      } else {
        const int per = hq / hkv;  // hkv divides hq without a map
        for (int h = hk * per; h < (hk + 1) * per; ++h)
          s.add_rows(base + static_cast<size_t>(h) * d, stride, r0, r1, slices);
      }
    }
    s.settle();
    reduce_slices(s, part_s, rs, cc, slices, d,
                  sq + ((static_cast<size_t>(b) * hkv + hk) * tm + u) * d);
  } else {
    const size_t stride = static_cast<size_t>(hkv) * d;
    const uint16_t* base =
        k + static_cast<size_t>(start) * stride + static_cast<size_t>(hk) * d + cc * 8;
    const int j0 = (u - tm) * gpc;
    for (int j = j0; j < min(j0 + gpc, kGroups); ++j) {
      if (active)
        s.add_rows(base, stride, j * keys_per_group + rs,
                   min((j + 1) * keys_per_group, len), slices);
      s.settle();
      reduce_slices(s, part_s, rs, cc, slices, d,
                    sk + ((static_cast<size_t>(b) * hkv + hk) * kGroups + j) * d);
      s.clear();
    }
  }
}

// One CTA per (sequence, KV head, run of kRankRows query-tile rows): the
// key groups' sums are staged once in shared memory as 24-bit limbs, then
// four rows at a time, 64 threads each: thread j computes the statistic of
// group j over all channels, with Sq = a1 * 2^24 + a0 and Sk = b1 * 2^24 +
// b0 (0 <= a0, b0 < 2^24),
//   Sq . Sk = 2^48 sum a1 b1 + 2^24 sum (a0 b1 + a1 b0) + sum a0 b0.
// The host admits only tiles with rows, keys < 2^15, rows * d and keys * d
// < 2^22 and rows * keys * d < 2^47 (rows = query rows of a tile times its
// query heads, keys = keys of a group), where |Sq| < 2^40 rows and |Sk| <
// 2^40 keys: the limbs fit int32, the three low sums int64 (their sum
// included), and the statistic int128.  Thread j then ranks group j, writes
// its byte, and warp ballots give the routing word.
constexpr int kRankRows = 4;
constexpr int kRankLanes = 4;  // rows in flight, 64 threads each
constexpr int kKPitch = kGroups + 1;  // int2 per channel row of the stage

__host__ __device__ constexpr int rank_smem_bytes(int d) {
  return d * kKPitch * static_cast<int>(sizeof(int2));
}

__device__ __forceinline__ int2 limbs24(int64_t v) {
  return make_int2(static_cast<int>(v & 0xFFFFFF), static_cast<int>(v >> 24));
}

__global__ void __launch_bounds__(64 * kRankLanes)
    rank_kernel(const int32_t* __restrict__ cu_seqlens,
                const int32_t* __restrict__ head_map, int hq, int max_seqlen,
                int total_tokens, int hkv, int tm, int d, int block_m,
                int block_n, int group, int permille,
                const int64_t* __restrict__ sq, const int64_t* __restrict__ sk,
                uint8_t* __restrict__ route, uint64_t* __restrict__ mask) {
  extern __shared__ int2 k_s[];  // [channel][kKPitch]: group j at column j
  __shared__ int2 q_s[kRankLanes][256];
  __shared__ __int128 imp_s[kRankLanes][kGroups];
  const int tid = threadIdx.x;
  const int rl = tid >> 6;  // row lane
  const int j = tid & 63;
  const int lane = tid & 31;
  const int chunks = (tm + kRankRows - 1) / kRankRows;
  const long long bh = blockIdx.x / chunks;  // b * hkv + hk
  const int m0 = static_cast<int>(blockIdx.x % chunks) * kRankRows;
  const int b = static_cast<int>(bh / hkv);
  const int start = cu_seqlens[b];
  const int len = cu_seqlens[b + 1] - start;
  // A head_map entry outside [0, hkv) makes the whole call invalid (the
  // first pass reported it and left that head out of every sum): every row
  // is then written as 0, like the rows of an invalid sequence.
  bool bad_map = false;
  if (head_map)
    for (int h = tid; h < hq; h += blockDim.x) {
      const int hm = head_map[h];
      bad_map |= hm < 0 || hm >= hkv;
    }
  bad_map = __syncthreads_or(bad_map) != 0;
  const bool seq_ok = !bad_map && start >= 0 && len >= 0 &&
                      len <= max_seqlen && start + len <= total_tokens;
  // key sums of the 64 groups, read along channels (coalesced, 16 bytes
  // per thread and eight loads in flight: 64 * d / 2 is a multiple of the
  // block size for d a multiple of 8)
  const longlong2* skb = reinterpret_cast<const longlong2*>(sk + bh * kGroups * d);
  const int n2 = kGroups * d / 2;
  for (int i0 = tid; i0 < n2; i0 += 8 * blockDim.x) {
    longlong2 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      v[u] = i < n2 ? __ldg(skb + i) : make_longlong2(0, 0);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < n2) {
        const int g = (2 * i) / d, c = 2 * i - g * d;
        k_s[c * kKPitch + g] = limbs24(v[u].x);
        k_s[(c + 1) * kKPitch + g] = limbs24(v[u].y);
      }
    }
  }
  for (int it = 0; it < kRankRows / kRankLanes; ++it) {
    const int m = m0 + it * kRankLanes + rl;
    const bool row_ok = m < tm;
    const long long row = bh * tm + m;
    int G = 0;  // an invalid sequence was reported by the first pass
    if (row_ok && seq_ok && static_cast<long long>(m) * block_m < len)
      G = ((min((m + 1) * block_m, len) - 1) / block_n) / group + 1;
    if (row_ok)
      for (int c = j; c < d; c += 64) q_s[rl][c] = limbs24(sq[row * d + c]);
    __syncthreads();
    if (j < G) {
      int64_t lo = 0, mid = 0;
      __int128 hi = 0;
#pragma unroll 4
      for (int c = 0; c < d; ++c) {
        const int2 a = q_s[rl][c];
        const int2 k = k_s[c * kKPitch + j];
        lo += static_cast<int64_t>(a.x) * k.x;
        mid += static_cast<int64_t>(a.x) * k.y + static_cast<int64_t>(a.y) * k.x;
        hi += static_cast<int64_t>(a.y) * k.y;
      }
      imp_s[rl][j] = (hi << 48) + (static_cast<__int128>(mid) << 24) + lo;
    }
    __syncthreads();
    const int k_fp16 = G - (permille * G + 500) / 1000;
    uint8_t bit = 0;
    if (j < G) {
      const __int128 v = imp_s[rl][j];
      int rank = 0;  // groups ahead of j: a larger statistic, or equal and smaller index
      for (int i = 0; i < G; ++i) {
        const __int128 x = imp_s[rl][i];
        rank += (x > v || (x == v && i < j)) ? 1 : 0;
      }
      bit = rank >= k_fp16 ? 1 : 0;
    }
    if (row_ok && route) route[row * 64 + j] = bit;
    const uint32_t half = __ballot_sync(0xffffffffu, bit != 0);
    if (row_ok && mask && lane == 0)
      reinterpret_cast<uint32_t*>(mask + row)[j >> 5] = half;
    __syncthreads();  // q_s and imp_s are rewritten by the next rows
  }
}

}  // namespace

// Scratch for tilemix_route_adaptive_noalloc: one instance per device
// context, reserved when this module loads, never allocated per call.  All
// calls on a device share it, so calls whose work overlaps on the device
// race on it (the declaration in tilemix.h says how to order them).
static __device__ __align__(256) unsigned char
    g_route_scratch[TILEMIX_ROUTE_ADAPTIVE_STATIC_BYTES];

// The array's address in the current context, looked up on every call (a
// host-side table lookup once the module is loaded): a cached address could
// outlive its context (a device reset, or another context on the same
// device) and send the kernels to memory that is no longer theirs.  In host
// code `g_route_scratch` names a host stand-in, never the device array.
cudaError_t route_adaptive_static_scratch(void** ptr) {
  return cudaGetSymbolAddress(ptr, g_route_scratch);
}

size_t route_adaptive_workspace(int batch, int max_seqlen, int hkv, int d,
                                int block_m) {
  const size_t tm = (static_cast<size_t>(max_seqlen) + block_m - 1) / block_m;
  return sizeof(int64_t) * d * static_cast<size_t>(batch) * hkv *
         (tm + kGroups);
}

cudaError_t launch_route_adaptive(const void* q, const void* k,
                                  const int32_t* cu_seqlens, int batch,
                                  int max_seqlen, int total_tokens, int hq,
                                  int hkv, int d,
                                  const int32_t* head_map, int block_m,
                                  int block_n, int group, int permille,
                                  void* workspace, uint8_t* route,
                                  uint64_t* mask, int32_t* status,
                                  cudaStream_t stream) {
  const int tm = (max_seqlen + block_m - 1) / block_m;
  int64_t* sq = static_cast<int64_t*>(workspace);
  int64_t* sk = sq + static_cast<size_t>(d) * batch * hkv * tm;
  // key CTAs take gpc consecutive groups, about 256 keys in all
  const int kpg = group * block_n;
  const int gpc = kpg >= 256 ? 1 : 256 / kpg;
  const dim3 g1(tm + (kGroups + gpc - 1) / gpc, hkv, batch);
  sums_kernel<<<g1, kSumThreads, 0, stream>>>(
      static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
      cu_seqlens, head_map, max_seqlen, total_tokens, hq, hkv, d, tm, block_m,
      kpg, gpc, sq, sk, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long ctas = static_cast<long long>(batch) * hkv *
                         ((tm + kRankRows - 1) / kRankRows);
  const int smem = rank_smem_bytes(d);
  e = cudaFuncSetAttribute(rank_kernel,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  rank_kernel<<<static_cast<unsigned>(ctas), 64 * kRankLanes, smem, stream>>>(
      cu_seqlens, head_map, hq, max_seqlen, total_tokens, hkv, tm, d, block_m,
      block_n, group, permille, sq, sk, route, mask);
  return cudaGetLastError();
}

}  // namespace tilemix
