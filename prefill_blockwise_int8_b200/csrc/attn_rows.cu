// Fused causal tile-routed FP16/INT8 prefill attention for sm_100a, with
// whole-row softmax warpgroups.
//
// Method: TileMix (arXiv 2608.17336).  Section 3 Preliminaries of the
// paperlayer summary: scores S = QK^T, online softmax keeping row maxima and
// normalisers, one 64-bit routing word per query-tile row whose bit
// floor(n/g) picks INT8 (Q8 K8^T, INT32 accumulation, rescaled by the block
// scales) or FP16 for key tile n; legality (causal, sequence end) decided
// separately from routing (appendix B).  Both paths update one shared
// online-softmax state and the FP16 P V product (ainews summary; appendix C).
//
// B200 design.  A CTA owns two 128-row query tiles of one head of one
// sequence (rows 256M .. 256M+255) and walks the 128-key tiles of their
// causal range; both tiles read every K / V tile once from shared memory.
//   warp 8      TMA producer: Q and / or Q8 of both tiles once, then per key
//               tile the K halves in each format some tile routes them to
//               (fp16 and / or int8, packed into a byte ring so an INT8-only
//               tile takes 16 KB, not 48) and the fp16 V tile;
//   warp 9      one thread issues tcgen05.mma: S_t = Q_t K^T (kind::f16, f32
//               in TMEM) or Q8_t K8^T (kind::i8, s32 in TMEM) per 64-key half
//               on its routed path (one N = 128 chain when both halves agree),
//               and O_t += P_t V with P_t read from TMEM (kind::f16, f32 O in
//               TMEM); each chain issues from precomputed descriptors;
//   warps 0-3   softmax of query tile 0, warps 4-7 of tile 1: one thread per
//               score row (= TMEM lane) owns the row's 128 scores, so the row
//               max, the exponentials and the row sum need no exchange with
//               other threads; one TMEM load round trip per tile;
//   warps 10-11 INT8 KV cache only: K8 -> fp16 K for FP16-routed halves and
//               V8 -> fp16 V on chip.
// The two tiles alternate on the tensor core: while one tile's softmax runs,
// the other tile's P V and next Q K^T execute.
#include <cuda.h>
#include <cuda_fp16.h>
#include <climits>
#include <math_constants.h>
#include <stdint.h>

#include "attn_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace tilemix {
namespace {

constexpr int kBM = 128;   // query rows per tile = TMEM lanes = MMA M
constexpr int kBN = 128;   // keys per compute tile
constexpr int kHalf = 64;  // routing granularity inside a compute tile
constexpr int kThreads = 384;
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;
constexpr int kWarpConv = 10;  // two converter warps (INT8 KV cache)
constexpr int kSmemBudget = 232448;
constexpr int kKRecs = 4;      // key tiles in flight in the K ring
constexpr int kVStages = 2;
// Registers: the block launches with kRegsLaunch per thread; the two softmax
// warpgroups take kRegsSoftmax and give the producer / MMA / converter
// warpgroup kRegsOther: 2 * 128 * 208 + 128 * 88 = 384 * 168.
constexpr int kRegsLaunch = 168, kRegsSoftmax = 208, kRegsOther = 88;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther <= kThreads * kRegsLaunch,
              "register split exceeds the launch allocation");

template <int D, bool KV8>
struct RowCfg {
  static constexpr int kQBytes = kBM * D * 2;   // fp16 Q of one tile
  static constexpr int kQ8Bytes = kBM * D;      // int8 Q8 of one tile
  static constexpr int kK16Half = kHalf * D * 2;  // fp16 K of 64 keys
  static constexpr int kK8Half = kHalf * D;       // int8 K8 of 64 keys
  static constexpr int kVBytes = kBN * D * 2;
  // INT8 V tile staged where the fp16 tile's last column chunk goes (d = 128:
  // row r of V8 lies where chunk 1 of row r of V goes; converted in place,
  // each row by the thread that read it); d = 64 stages it past the tile.
  static constexpr int kV8Bytes = kBN * D;
  static constexpr int kV8Off = D == 128 ? kVBytes - kV8Bytes : kVBytes;
  static constexpr int kVSlot = (KV8 && D != 128) ? kVBytes + kV8Bytes : kVBytes;
  static constexpr int kQ8Off = 2 * kQBytes;
  static constexpr int kKRing = 2 * kQBytes + 2 * kQ8Bytes;
  static constexpr int kKRingBytes = 65536;  // a power of two
  static constexpr int kVRing = kKRing + kKRingBytes;
  static constexpr int kBarOff = kVRing + kVStages * kVSlot;
  // barrier indices
  static constexpr int kBarQ = 0;
  static constexpr int kBarKFull = 1;
  static constexpr int kBarKEmpty = kBarKFull + kKRecs;
  static constexpr int kBarKConv = kBarKEmpty + kKRecs;
  static constexpr int kBarVFull = kBarKConv + kKRecs;
  static constexpr int kBarVEmpty = kBarVFull + kVStages;
  static constexpr int kBarVConv = kBarVEmpty + kVStages;
  static constexpr int kBarS = kBarVConv + kVStages;  // [tile]
  static constexpr int kBarP = kBarS + 2;             // [tile]
  static constexpr int kBarO = kBarP + 2;             // [tile]
  static constexpr int kBarOStage = kBarO + 2;        // [tile]
  static constexpr int kBarDrain = kBarOStage + 2;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kBarBytes = 512;
  static_assert(kNumBars * 8 + 16 <= kBarBytes, "barrier area");
  static constexpr int kSmem = kBarOff + kBarBytes + 1024;  // + align slack
  static_assert(kSmem <= kSmemBudget, "shared memory overflow");
  // TMEM: S_t at t * 256 (128 columns, P over its first 64), O_t after it
  static constexpr int kTileCols = 256;
  static constexpr int kOCol = 128;
  static_assert(kOCol + D <= kTileCols, "TMEM overflow");
};

// Where the K halves of one key tile sit in the K ring: pos16 / pos8 are
// byte offsets (-1: not loaded) of the fp16 / int8 block, h16 / h8 the
// halves each block holds (3: both, a 128-key block; 1 or 2: that half
// alone, a 64-key block).
struct KRec {
  int pos16, pos8;
  uint32_t h16, h8;
};

// The K ring's allocator.  Producer, MMA issuer and converters run the same
// sequence of plans, so they agree on every position without talking; a
// block never wraps (it skips to the ring's start instead).
template <int D, int RING>
struct KRing {
  uint32_t head = 0;  // bytes handed out so far, skipped tails included
  __device__ __forceinline__ int place(int bytes) {
    uint32_t off = head & (RING - 1);
    if (off + bytes > RING) {
      head += RING - off;
      off = 0;
    }
    head += bytes;
    return static_cast<int>(off);
  }
  __device__ __forceinline__ KRec plan(uint32_t h16, uint32_t h8) {
    KRec r{-1, -1, h16, h8};
    constexpr int k16h = kHalf * D * 2, k8h = kHalf * D;
    if (h16) r.pos16 = place(h16 == 3u ? 2 * k16h : k16h);
    if (h8) r.pos8 = place(h8 == 3u ? 2 * k8h : k8h);
    return r;
  }
};

// Routing state of one 128-row query tile.
struct RowTile {
  uint64_t w;   // routing word of its 128 rows
  int nl;       // last legal 64-key block of the tile (-1: no rows)
  int n_last;   // last legal 128-key tile (-1: no rows)
};

__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Largest score of the 64-key half sv[j0 .. j0+63] held as raw TMEM bits
// (INT32 accumulators when I8, fp32 otherwise), scaled by c >= 0 into the
// log2 domain; with MASKED, columns j > hl (relative to j0) are left out and
// a half with no legal column gives -inf.  Scaling by c >= 0 keeps the
// order, so only the maximum is converted.
template <bool I8, bool MASKED>
__device__ __forceinline__ float half_max(const uint32_t (&sv)[128], int j0,
                                          int hl, float c) {
  if (MASKED && hl < 0) return -CUDART_INF_F;
  if (I8) {
    auto g = [&](int j) {
      return (!MASKED || j <= hl) ? static_cast<int>(sv[j0 + j]) : INT_MIN;
    };
    int a[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = max(g(2 * k), g(2 * k + 1));
#pragma unroll
    for (int j = 16; j < 64; j += 16)
#pragma unroll
      for (int k = 0; k < 8; ++k)
        a[k] = __vimax3_s32(a[k], g(j + 2 * k), g(j + 2 * k + 1));
    const int m = __vimax3_s32(__vimax3_s32(a[0], a[1], a[2]),
                               __vimax3_s32(a[3], a[4], a[5]), max(a[6], a[7]));
    return __int2float_rn(m) * c;
  } else {
    auto g = [&](int j) {
      return (!MASKED || j <= hl) ? __uint_as_float(sv[j0 + j]) : -CUDART_INF_F;
    };
    float a[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = fmaxf(g(2 * k), g(2 * k + 1));
#pragma unroll
    for (int j = 16; j < 64; j += 16)
#pragma unroll
      for (int k = 0; k < 8; ++k)
        a[k] = fmax3f(a[k], g(j + 2 * k), g(j + 2 * k + 1));
    return fmax3f(fmax3f(a[0], a[1], a[2]), fmax3f(a[3], a[4], a[5]),
                  fmaxf(a[6], a[7])) * c;
  }
}

// P of a 32-key chunk held as raw TMEM bits in sv: 2^(s c - m) rounded to
// fp16, packed in pairs (key 2i in the low half of pk[i]); the same rounded
// values are added to the partial sums, so O / l is a weighted mean with
// exactly the weights P V uses.  INT32 scores convert exactly (|acc| <=
// 127^2 d < 2^24) inside the same pass.  With MASKED, columns j > hl give 0.
template <bool I8, bool MASKED>
__device__ __forceinline__ void chunk_exp(const uint32_t (&sv)[32], float c,
                                          float m, int hl, uint32_t (&pk)[16],
                                          float2& sa, float2& sb) {
  const float2 c2 = make_float2(c, c);
  const float2 nm2 = make_float2(-m, -m);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int j = 2 * i;
    float2 v;
    if (I8) {
      v = make_float2(__int2float_rn(static_cast<int>(sv[j])),
                      __int2float_rn(static_cast<int>(sv[j + 1])));
    } else {
      v = make_float2(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1]));
    }
    float2 e = __ffma2_rn(v, c2, nm2);
    if (MASKED) {  // 2^-inf = 0, also when c == 0
      e.x = (j <= hl) ? e.x : -CUDART_INF_F;
      e.y = (j + 1 <= hl) ? e.y : -CUDART_INF_F;
    }
    const __half2 ph = __floats2half2_rn(ex2_approx(e.x), ex2_approx(e.y));
    const float2 pr = __half22float2(ph);
    if (i & 1) sb = __fadd2_rn(sb, pr);
    else sa = __fadd2_rn(sa, pr);
    pk[i] = *reinterpret_cast<const uint32_t*>(&ph);
  }
}

// Masked tiles (the diagonal and the sequence end): the same work with the
// causal / end mask, kept out of line so the unmasked loop stays small in
// the instruction cache.  Row max of the 128 scores at s_addr (TMEM), with
// columns j > hl left out.
__device__ __noinline__ float masked_row_max(uint32_t s_addr, bool i80,
                                             bool i81, float c0, float c1,
                                             int hl) {
  uint32_t sv[128];
  tmem_ld32_at(s_addr, sv, 0);
  tmem_ld32_at(s_addr, sv, 32);
  tmem_ld32_at(s_addr, sv, 64);
  tmem_ld32_at(s_addr, sv, 96);
  tmem_ld_wait();
  const float m0 = i80 ? half_max<true, true>(sv, 0, hl, c0)
                       : half_max<false, true>(sv, 0, hl, c0);
  const float m1 = i81 ? half_max<true, true>(sv, 64, hl - 64, c1)
                       : half_max<false, true>(sv, 64, hl - 64, c1);
  return fmaxf(m0, m1);
}

// P of the 32-key chunk at s_addr with columns j > hl masked, stored as 16
// fp16 pairs at p_addr; returns the chunk's row sum of the rounded P.
__device__ __noinline__ float masked_chunk_exp(uint32_t s_addr, uint32_t p_addr,
                                               bool i8, float c, float m,
                                               int hl) {
  uint32_t s32[32], pk[16];
  tmem_ld32(s_addr, s32);
  tmem_ld_wait();
  float2 sa = make_float2(0.f, 0.f), sb = sa;
  if (i8) chunk_exp<true, true>(s32, c, m, hl, pk, sa, sb);
  else chunk_exp<false, true>(s32, c, m, hl, pk, sa, sb);
  tmem_st16(p_addr, pk);
  const float2 cs = __fadd2_rn(sa, sb);
  return cs.x + cs.y;
}

// O *= alpha (per row) for the D columns of O in TMEM at `o_addr`; a rare
// path (the running max grew by more than 2^8), kept out of the hot loop.
template <int D>
__device__ __noinline__ void rescale_o(uint32_t o_addr, float alpha) {
#pragma unroll 1
  for (int oc = 0; oc < D; oc += 32) {
    uint32_t o[32];
    tmem_ld32(o_addr + oc, o);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 32; ++j)
      o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
    tmem_st32(o_addr + oc, o);
  }
  tmem_st_wait();
}

// Test output: the raw INT32 scores of this row's 64-key half at `col`
// (TMEM columns) to dst[0 .. keys_left); warp-collective loads, per-thread
// stores (`store` false for rows past the sequence).
__device__ __noinline__ void dump_half(uint32_t s_addr, int32_t* dst,
                                       int keys_left, bool store) {
  uint32_t v[32];
#pragma unroll 1
  for (int q = 0; q < 2; ++q) {
    tmem_ld32(s_addr + 32 * q, v);
    tmem_ld_wait();
    if (store)
      for (int j = 0; j < 32; ++j)
        if (32 * q + j < keys_left) dst[32 * q + j] = static_cast<int32_t>(v[j]);
  }
}

template <int D, bool KV8>
__global__ void __launch_bounds__(kThreads, 1)
    attn_rows_kernel(const __grid_constant__ AttnParams p) {
  using C = RowCfg<D, KV8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Grid (head, query-tile pair, sequence); longest pairs first.
  const int h = blockIdx.x;
  const int mp = gridDim.y - 1 - blockIdx.y;
  const int b = blockIdx.z;

  // A status word that already holds an error stops every later CTA.
  if (p.status && *reinterpret_cast<volatile int32_t*>(p.status) != 0) return;

  const int start = p.cu_seqlens[b];
  const int len = p.cu_seqlens[b + 1] - start;
  if (start < 0 || len < 0 || len > p.max_seqlen ||
      start + len > p.total_tokens) {
    if (threadIdx.x == 0) report_status(p.status, kStatusBadSeqlens);
    return;
  }
  const int row_base = mp * (2 * kBM);
  if (row_base >= len) return;
  const int hk = p.head_map ? p.head_map[h] : h / p.heads_per_kv;
  if (hk < 0 || hk >= p.hkv) {
    if (threadIdx.x == 0) report_status(p.status, kStatusBadSeqlens);
    return;
  }

  const bool routed = !p.fp16_only;
  const size_t wbase = (static_cast<size_t>(b) * p.hkv + hk) * p.tm_route;
  auto tile_of = [&](int t) {
    const int row0 = row_base + t * kBM;
    RowTile r{0ull, -1, -1};
    if (row0 < len) {
      const int last = min(row0 + kBM - 1, len - 1);
      r.n_last = last / kBN;
      r.nl = last / kHalf;
      r.w = routed ? p.mask[wbase + row0 / kBM] : 0ull;
    }
    return r;
  };
  const RowTile rt0 = tile_of(0), rt1 = tile_of(1);
  // Per-tile values by selection, never through a reference: a reference
  // to a local struct would put it in local memory on the hot paths.
  auto w_of = [&](int t) { return t ? rt1.w : rt0.w; };
  auto nl_of = [&](int t) { return t ? rt1.nl : rt0.nl; };
  auto last_of = [&](int t) { return t ? rt1.n_last : rt0.n_last; };
  const int n_end = max(rt0.n_last, rt1.n_last);
  const int tpb = p.tiles_per_bit;  // 64-key blocks per routing bit
  // Path of 64-key half kh of key tile n for query tile t (0: no legal key).
  auto kind_of = [&](int t, int n, int kh) -> uint32_t {
    const int n64 = 2 * n + kh;
    if (n64 > nl_of(t)) return 0u;
    return ((w_of(t) >> (n64 / tpb)) & 1ull) ? kKindI8 : kKindF16;
  };
  // K halves of key tile n that some query tile needs, per format.  The
  // INT8 cache always brings the whole K8 tile (the fp16 copy is made from
  // it on chip).
  // Returned packed (h16 | h8 << 2), by value.
  auto halves_of = [&](int n) -> uint32_t {
    uint32_t h16 = 0u, h8 = 0u;
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int kh = 0; kh < 2; ++kh) {
        const uint32_t k = kind_of(t, n, kh);
        if (k == kKindF16) h16 |= 1u << kh;
        if (k == kKindI8) h8 |= 1u << kh;
      }
    if (KV8) h8 = 3u;
    return h16 | (h8 << 2);
  };

  // ---- shared memory ----
  auto sQ = [&](int t) { return smem + t * C::kQBytes; };
  auto sQ8 = [&](int t) { return smem + C::kQ8Off + t * C::kQ8Bytes; };
  uint8_t* kring = smem + C::kKRing;
  auto vslot = [&](int s) { return smem + C::kVRing + s * C::kVSlot; };
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (warp == kWarpProducer && lane == 0) {
    mbar_init(&bars[C::kBarQ], 1);
    for (int s = 0; s < kKRecs; ++s) {
      mbar_init(&bars[C::kBarKFull + s], 1);
      mbar_init(&bars[C::kBarKEmpty + s], 1);
      mbar_init(&bars[C::kBarKConv + s], 2);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bars[C::kBarVFull + s], 1);
      mbar_init(&bars[C::kBarVEmpty + s], 1);
      mbar_init(&bars[C::kBarVConv + s], 2);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars[C::kBarS + t], 1);
      mbar_init(&bars[C::kBarP + t], 4);       // one arrival per softmax warp
      mbar_init(&bars[C::kBarO + t], 1);
      mbar_init(&bars[C::kBarOStage + t], 4);  // O of tile t staged
    }
    mbar_init(&bars[C::kBarDrain], 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_o);
    if (KV8) {
      tma_prefetch_desc(&p.tm_kh8);
      tma_prefetch_desc(&p.tm_v8);
    } else {
      tma_prefetch_desc(&p.tm_kh);
      tma_prefetch_desc(&p.tm_v);
      if (routed) tma_prefetch_desc(&p.tm_kh8);
    }
    if (routed) tma_prefetch_desc(&p.tm_q8);
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&]() {
    *abort_flag = 1;
    report_status(p.status, kStatusTimeout);
  };

  if (warp >= 8) {
  regs_dec<kRegsOther>();
  if (warp == kWarpProducer) {
    // =================== TMA producer ===================
    if (lane == 0) {
      // Formats a query tile uses anywhere: its word's bits over the legal
      // groups (bit set: INT8 somewhere; bit clear: FP16 somewhere).
      auto need_of = [&](const RowTile& r) -> uint32_t {
        if (r.nl < 0) return 0u;
        const int gl = r.nl / tpb;  // last legal group
        const uint64_t legal = gl >= 63 ? ~0ull : ((1ull << (gl + 1)) - 1ull);
        uint32_t k = 0;
        if (r.w & legal) k |= kKindI8;
        if (~r.w & legal) k |= kKindF16;
        return k;
      };
      uint32_t qbytes = 0;
      const uint32_t need[2] = {need_of(rt0), need_of(rt1)};
      for (int t = 0; t < 2; ++t)
        qbytes += ((need[t] & kKindF16) ? C::kQBytes : 0) +
                  ((need[t] & kKindI8) ? C::kQ8Bytes : 0);
      mbar_arrive_expect_tx(&bars[C::kBarQ], qbytes);
      for (int t = 0; t < 2; ++t) {
        const int qrow = start + row_base + t * kBM;
        if (need[t] & kKindF16)
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sQ(t) + c * kBM * 128, &p.tm_q, &bars[C::kBarQ],
                        c * 64, qrow, h);
        if (need[t] & kKindI8)
          tma_load_3d(sQ8(t), &p.tm_q8, &bars[C::kBarQ], 0, qrow, h);
      }
      KRing<D, C::kKRingBytes> ring;
      uint32_t rec_end[kKRecs];
      uint32_t freed = 0;
      int oldest = 0;  // oldest key tile whose K blocks may still be read
      int k_issued = 0, v_issued = 0;
      bool v_withheld = false;
      bool ok = true;
      for (int n = 0; n <= n_end && ok; ++n) {
        const int krow = start + n * kBN;
        const uint32_t hh = halves_of(n);
        const uint32_t h16 = hh & 3u, h8 = hh >> 2;
        const KRec rec = ring.plan(h16, h8);
        // Room in the ring and a free record: wait for the oldest tiles'
        // Q K^T to finish reading their blocks.  Live blocks span
        // [freed, head) of the allocation count; once no older tile is live
        // the ring is empty and the new tile fits whatever it skipped.
        while (ok && (n - oldest >= kKRecs ||
                      (oldest < n && ring.head - freed > C::kKRingBytes))) {
          if (!mbar_wait(&bars[C::kBarKEmpty + oldest % kKRecs],
                         (oldest / kKRecs) & 1, abort_flag)) {
            ok = false;
            break;
          }
          freed = rec_end[oldest % kKRecs];
          ++oldest;
        }
        if (!ok) break;
        rec_end[n % kKRecs] = ring.head;
        const int ks = n % kKRecs;
        // fp16 K: converted on chip from K8 with the INT8 cache
        const uint32_t b16 = KV8 ? 0u : (h16 == 3u ? 2 : (h16 ? 1 : 0)) * C::kK16Half;
        const uint32_t b8 = (h8 == 3u ? 2 : (h8 ? 1 : 0)) * C::kK8Half;
        mbar_arrive_expect_tx(&bars[C::kBarKFull + ks], b16 + b8);
        if (!KV8 && h16) {
          // [D/64 chunks][rows][128 B]; a 64-key block holds only its half
          const int rows = h16 == 3u ? kBN : kHalf;
          for (int c = 0; c < D / 64; ++c)
            for (int r = 0; r < 2; ++r) {
              if (!((h16 >> r) & 1u)) continue;
              const int dst_row = h16 == 3u ? r * kHalf : 0;
              tma_load_3d(kring + rec.pos16 + c * rows * 128 + dst_row * 128,
                          &p.tm_kh, &bars[C::kBarKFull + ks], c * 64,
                          krow + r * kHalf, hk);
            }
        }
        if (h8)
          for (int r = 0; r < 2; ++r) {
            if (!((h8 >> r) & 1u)) continue;
            const int dst_row = h8 == 3u ? r * kHalf : 0;
            tma_load_3d(kring + rec.pos8 + dst_row * D, &p.tm_kh8,
                        &bars[C::kBarKFull + ks], 0, krow + r * kHalf, hk);
          }
        k_issued = n + 1;
        // V tile n
        const int vs = n % kVStages;
        const int jv = n / kVStages;
        if (jv > 0 &&
            !mbar_wait(&bars[C::kBarVEmpty + vs], (jv - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        // Timeout-path test: V tile 0 is never loaded, so its barrier never
        // completes and the MMA issuer's bounded wait on it expires.
        if (n == 0 && p.test_expire_wait) {
          v_withheld = true;
          continue;
        }
        if (KV8) {
          mbar_arrive_expect_tx(&bars[C::kBarVFull + vs], C::kV8Bytes);
          tma_load_3d(vslot(vs) + C::kV8Off, &p.tm_v8, &bars[C::kBarVFull + vs],
                      0, krow, hk);
        } else {
          mbar_arrive_expect_tx(&bars[C::kBarVFull + vs], C::kVBytes);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(vslot(vs) + c * kBN * 128, &p.tm_v,
                        &bars[C::kBarVFull + vs], c * 64, krow, hk);
        }
        v_issued = n + 1;
      }
      if (!ok) {
        fail();
        // Let the copies already in flight land before the CTA exits.
        mbar_wait(&bars[C::kBarQ], 0, nullptr);
        for (int n = max(0, k_issued - kKRecs); n < k_issued; ++n)
          mbar_wait(&bars[C::kBarKFull + n % kKRecs], (n / kKRecs) & 1, nullptr);
        for (int n = max(0, v_issued - kVStages); n < v_issued; ++n)
          if (!(n == 0 && v_withheld))
            mbar_wait(&bars[C::kBarVFull + n % kVStages], (n / kVStages) & 1,
                      nullptr);
      }
    }
  } else if (warp == kWarpMma) {
    // =================== MMA issuer (one thread) ===================
    if (lane == 0) {
      constexpr uint32_t id16_full = instr_desc(1, 0, 0, 0, 0, kBN, kBM);
      constexpr uint32_t id16_half = instr_desc(1, 0, 0, 0, 0, kHalf, kBM);
      constexpr uint32_t id8_full = instr_desc(2, 1, 1, 0, 0, kBN, kBM);
      constexpr uint32_t id8_half = instr_desc(2, 1, 1, 0, 0, kHalf, kBM);
      constexpr uint32_t idesc_pv = instr_desc(1, 0, 0, 0, 1, D, kBM);
      bool ok = mbar_wait(&bars[C::kBarQ], 0, abort_flag);
      tc_fence_after();
      // base descriptors of the resident Q / Q8 tiles (K-step 0)
      const uint64_t dq16_0 = desc_k_f16(smem_u32(sQ(0)), kBM * 128, 0);
      const uint64_t dq16_1 = desc_k_f16(smem_u32(sQ(1)), kBM * 128, 0);
      const uint64_t dq8_0 = desc_k_i8<D>(smem_u32(sQ8(0)), 0);
      const uint64_t dq8_1 = desc_k_i8<D>(smem_u32(sQ8(1)), 0);
      const uint32_t kring_u32 = smem_u32(kring);
      // S_t = Q_t K(n)^T, each 64-key half on its path.  A half no row of
      // tile t can see takes the other half's path when that format's block
      // covers it (one N = 128 chain), else it is skipped.
      auto issue_qk = [&](int t, int n, const KRec rec) {
        const uint32_t k0 = kind_of(t, n, 0);
        uint32_t k1 = kind_of(t, n, 1);
        if (k1 == 0u && ((k0 == kKindF16 && rec.h16 == 3u) ||
                         (k0 == kKindI8 && rec.h8 == 3u)))
          k1 = k0;
        const uint32_t halves16 = ((k0 == kKindF16) ? 1u : 0u) | ((k1 == kKindF16) ? 2u : 0u);
        const uint32_t halves8 = ((k0 == kKindI8) ? 1u : 0u) | ((k1 == kKindI8) ? 2u : 0u);
        const uint32_t tb = tmem + t * C::kTileCols;
        if (halves16) {
          // fp16 K block: D/64 chunks of [rows][128 B]
          const int rows = rec.h16 == 3u ? kBN : kHalf;
          const uint32_t hoff = (halves16 == 2u) ? 1u : 0u;
          const uint32_t base = kring_u32 + rec.pos16 +
                                (rec.h16 == 3u ? hoff * (kHalf * 128) : 0u);
          const uint64_t db0 = smem_desc(base, 16, 1024, kSwizzle128);
          const uint64_t db1 = smem_desc(base + rows * 128, 16, 1024, kSwizzle128);
          const uint64_t da0 = t ? dq16_1 : dq16_0;
          const uint64_t da1 = da0 + ((kBM * 128) >> 4);
          const uint32_t d = tb + hoff * kHalf;
          const uint32_t id = halves16 == 3u ? id16_full : id16_half;
          // compact loops: this code runs once per tile and must stay small
          // enough to survive in the instruction cache between tiles
#pragma unroll 1
          for (int c = 0; c < D / 64; ++c) {
            uint64_t a = c ? da1 : da0, bb = c ? db1 : db0;
#pragma unroll 1
            for (int k = 0; k < 4; ++k, a += 2, bb += 2)
              mma_f16_ss(d, a, bb, id, (c | k) ? 1u : 0u);
          }
        }
        if (halves8) {
          const uint32_t hoff = (halves8 == 2u) ? 1u : 0u;
          const uint32_t base = kring_u32 + rec.pos8 +
                                (rec.h8 == 3u ? hoff * (kHalf * D) : 0u);
          const uint64_t db = desc_k_i8<D>(base, 0);
          const uint64_t da = t ? dq8_1 : dq8_0;
          const uint32_t d = tb + hoff * kHalf;
          const uint32_t id = halves8 == 3u ? id8_full : id8_half;
          uint64_t a = da, bb = db;
#pragma unroll 1
          for (int ks = 0; ks < D / 32; ++ks, a += 2, bb += 2)
            mma_i8_ss(d, a, bb, id, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars[C::kBarS + t]);
      };
      // O_t += P_t(n) V(n), P_t(n) in the first 64 columns of S_t.
      auto issue_pv = [&](int t, int n, uint64_t dv) {
        const uint32_t tb = tmem + t * C::kTileCols;
        uint32_t acc = n > 0 ? 1u : 0u;
        uint32_t pa = tb;
#pragma unroll 1
        for (int ks = 0; ks < kBN / 16; ++ks, pa += 8, dv += 16 * 128 / 16) {
          mma_f16_ts(tb + C::kOCol, pa, dv, idesc_pv, acc);
          acc = 1u;
        }
      };
      auto wait_k = [&](int n) -> bool {
        const int s = n % kKRecs;
        const uint32_t ph = (n / kKRecs) & 1;
        if (!mbar_wait(&bars[C::kBarKFull + s], ph, abort_flag)) return false;
        // with the INT8 cache, the converters' fp16 K (they waited for the
        // TMA; the slot frees only after they passed it)
        if (KV8 && !mbar_wait(&bars[C::kBarKConv + s], ph, abort_flag))
          return false;
        tc_fence_after();
        return true;
      };

      KRing<D, C::kKRingBytes> ring;
      KRec rec_next{-1, -1, 0u, 0u};
      {
        const uint32_t hh = halves_of(0);
        const uint32_t h16 = hh & 3u, h8 = hh >> 2;
        rec_next = ring.plan(h16, h8);
      }
      if (ok) ok = wait_k(0);
      if (ok) {
        for (int t = 0; t < 2; ++t)
          if (last_of(t) >= 0) issue_qk(t, 0, rec_next);
        mma_commit(&bars[C::kBarKEmpty + 0]);
      }
      for (int n = 0; n <= n_end && ok; ++n) {
        KRec rec_n1{-1, -1, 0u, 0u};
        if (n + 1 <= n_end) {
          const uint32_t hh = halves_of(n + 1);
          const uint32_t h16 = hh & 3u, h8 = hh >> 2;
          rec_n1 = ring.plan(h16, h8);
        }
        const int vs = n % kVStages;
        bool v_ready = false, k_ready = false;
        for (int t = 0; t < 2 && ok; ++t) {
          if (n <= last_of(t)) {
            if (!mbar_wait(&bars[C::kBarP + t], n & 1, abort_flag)) {
              ok = false;
              break;
            }
            if (!v_ready) {
              // the INT8 cache: the converters' fp16 V
              if (!mbar_wait(&bars[(KV8 ? C::kBarVConv : C::kBarVFull) + vs],
                             (n / kVStages) & 1, abort_flag)) {
                ok = false;
                break;
              }
              v_ready = true;
            }
            tc_fence_after();
            issue_pv(t, n, desc_v(smem_u32(vslot(vs)), kBN * 128, 0));
            if (n == last_of(t)) mma_commit(&bars[C::kBarO + t]);
          }
          if (n + 1 <= last_of(t)) {
            if (!k_ready) {
              if (!wait_k(n + 1)) {
                ok = false;
                break;
              }
              k_ready = true;
            }
            issue_qk(t, n + 1, rec_n1);
          }
        }
        if (!ok) break;
        mma_commit(&bars[C::kBarVEmpty + vs]);
        if (n + 1 <= n_end) mma_commit(&bars[C::kBarKEmpty + (n + 1) % kKRecs]);
      }
      if (!ok) fail();
      // Drain: every MMA issued above has finished once this completes.
      mma_commit(&bars[C::kBarDrain]);
      mbar_wait(&bars[C::kBarDrain], 0, nullptr);
    }
    __syncwarp();
  } else if (warp >= kWarpConv) {
    // =================== INT8 KV cache converters (2 warps) ===================
    // Per key tile: K8 -> fp16 K (exact) for the halves some query tile
    // routes to FP16, and V8 -> fp16 v8 * 2^e.  Each thread converts whole
    // key rows, reading a row before writing it, which makes the in-place
    // V conversion safe.
    if (KV8) {
      const int ct = (warp - kWarpConv) * 32 + lane;
      const float* vscale =
          p.v_scale + (static_cast<size_t>(hk) * p.batch + b) * p.nbk;
      constexpr uint32_t k8_swz = D == 128 ? 7u : 3u;
      KRing<D, C::kKRingBytes> ring;
      bool ok = true;
      for (int n = 0; n <= n_end && ok; ++n) {
        const uint32_t hh = halves_of(n);
        const uint32_t h16 = hh & 3u, h8 = hh >> 2;
        const KRec rec = ring.plan(h16, h8);
        const int ks = n % kKRecs;
        const bool got_k = mbar_wait(&bars[C::kBarKFull + ks],
                                     (n / kKRecs) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, got_k)) {
          ok = false;
          break;
        }
        if (h16) {
          const uint8_t* k8 = kring + rec.pos8;  // the whole K8 tile
          uint8_t* k16 = kring + rec.pos16;
          if (h16 == 3u) {
            for (int rr = ct; rr < kBN; rr += 64)
              convert_row<D, false, kBN * 128>(k8, k8_swz, k16, rr,
                                               __float2half2_rn(1.0f));
          } else {
            // a 64-key block of the half that needs it
            const int hh = h16 == 2u ? 1 : 0;
            convert_row<D, false, kHalf * 128>(k8 + hh * kHalf * D, k8_swz,
                                               k16, ct, __float2half2_rn(1.0f));
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[C::kBarKConv + ks]);

        const int vs = n % kVStages;
        const bool got_v = mbar_wait(&bars[C::kBarVFull + vs],
                                     (n / kVStages) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, got_v)) {
          ok = false;
          break;
        }
        uint8_t* vslot_p = vslot(vs);
        for (int rr = ct; rr < kBN; rr += 64) {
          // V scale sv = 2^e2 f with f in [1, 2): the fp16 tile holds
          // v8 2^e2 exactly (never above |v8 sv|); the softmax multiplies P
          // by f.
          const int blk = (n * kBN + rr) / p.quant_block_k;
          const float sv = vscale[min(blk, p.nbk - 1)];
          int e = 0;
          frexpf(sv, &e);
          const float pow2 = sv > 0.0f ? ldexpf(1.0f, e - 1) : 0.0f;
          convert_row<D, true, kBN * 128>(vslot_p + C::kV8Off, 0u, vslot_p, rr,
                                          __float2half2_rn(pow2));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[C::kBarVConv + vs]);
      }
      if (!ok) fail();
    }
  }
  } else {
    regs_inc<kRegsSoftmax>();
    // =================== softmax warps 0-7 ===================
    // Warpgroup t serves query tile t; thread = score row = TMEM lane, and
    // each thread holds its row's 128 scores of a key tile at once.
    const int t = warp >> 2;
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const RowTile R = t ? rt1 : rt0;  // by value
    bool ok = true;
    if (R.n_last >= 0) {
      const int r_local = row_base + t * kBM + r;
      const int key_lim = min(r_local, len - 1);  // keys j <= key_lim legal
      const uint32_t lane_addr = tmem + t * C::kTileCols + lane_off;
      const float* kscale =
          (routed || KV8)
              ? p.k_scale + (static_cast<size_t>(hk) * p.batch + b) * p.nbk
              : nullptr;
      auto ksc = [&](int n, int kh) {
        const int blk = (n * kBN + kh * kHalf) / p.quant_block_k;
        return kscale[min(blk, p.nbk - 1)];
      };
      // INT8 KV cache: the V scale's mantissa factor f in [1, 2) of a
      // 64-key half (the converters put its power of two into V).
      const float* vscale =
          KV8 ? p.v_scale + (static_cast<size_t>(hk) * p.batch + b) * p.nbk
              : nullptr;
      auto vfrac = [&](int n, int kh) {
        const int blk = (n * kBN + kh * kHalf) / p.quant_block_k;
        const float sv = vscale[min(blk, p.nbk - 1)];
        int e = 0;
        frexpf(sv, &e);
        return sv > 0.0f ? ldexpf(sv, 1 - e) : 1.0f;
      };
      // softmax scale (log2 units) times this row's Q block scale: the INT8
      // path's S c = (Q8 K8^T) sq sk scale log2(e)
      const float cq =
          routed ? p.scale_log2 *
                       p.q_scale[(static_cast<size_t>(h) * p.batch + b) * p.nbq +
                                 key_lim / p.quant_block_q]
                 : 0.0f;
      float m_run = -CUDART_INF_F, l_run = 0.0f;
      float sk0 = 0.0f, sk1 = 0.0f;
      if ((routed || KV8) && R.n_last >= 0) {
        sk0 = ksc(0, 0);
        sk1 = ksc(0, 1);
      }
      for (int n = 0; n <= R.n_last && ok; ++n) {
        const float c_sk0 = sk0, c_sk1 = sk1;
        if ((routed || KV8) && n < R.n_last) {  // next tile's, while waiting
          sk0 = ksc(n + 1, 0);
          sk1 = ksc(n + 1, 1);
        }
        float fv0 = 1.0f, fv1 = 1.0f;
        if (KV8) {
          fv0 = vfrac(n, 0);
          fv1 = vfrac(n, 1);
        }
        // Exits stay warp-uniform: the tcgen05.ld/st below are .sync.aligned.
        const bool got_s = mbar_wait(&bars[C::kBarS + t], n & 1, abort_flag);
        if (!__all_sync(0xffffffffu, got_s)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sv[128];
        tmem_ld32_at(lane_addr, sv, 0);
        tmem_ld32_at(lane_addr, sv, 32);
        tmem_ld32_at(lane_addr, sv, 64);
        tmem_ld32_at(lane_addr, sv, 96);
        tmem_ld_wait();
        // Path of each 64-key half: the tile's routing (all 128 rows share
        // one word); keys past every row of the tile are masked below.
        const bool i80 = kind_of(t, n, 0) == kKindI8;
        const bool i81 = kind_of(t, n, 1) == kKindI8 ||
                         (kind_of(t, n, 1) == 0u && i80);
        if (p.qk_dump) {
          for (int kh = 0; kh < 2; ++kh) {
            const int n64 = 2 * n + kh;
            if (!(kh ? i81 : i80) || n64 > R.nl) continue;  // uniform
            const int rr_all = min(r_local, len - 1);  // rows past len store nothing
            const int rrow = rr_all / p.route_bm;
            const int rr = rr_all - rrow * p.route_bm;
            const int key0 = n64 * kHalf;
            const int nr = key0 / p.route_bn;
            int32_t* dst =
                p.qk_dump +
                ((((static_cast<size_t>(b) * p.hq + h) * p.tm_route + rrow) *
                      p.tn_max +
                  nr) *
                     p.route_bm +
                 rr) *
                    p.route_bn +
                (key0 - nr * p.route_bn);
            dump_half(lane_addr + kh * kHalf, dst, len - key0, r_local < len);
          }
        }
        // score scale per half: INT8 sq sk scale log2(e); FP16 scale
        // log2(e) (the INT8 cache's fp16 K is k8, so sk joins)
        const float c0 = i80 ? cq * c_sk0 : (KV8 ? p.scale_log2 * c_sk0 : p.scale_log2);
        const float c1 = i81 ? cq * c_sk1 : (KV8 ? p.scale_log2 * c_sk1 : p.scale_log2);
        const int hl = key_lim - n * kBN;  // legal columns: j <= hl
        // The path of a half is the same for every row of the tile (one
        // routing word), so these branches are uniform across the warp.
        // The masked path loads from TMEM itself (warp-collective
        // tcgen05.ld), so the choice is made per warp: a warp with any
        // masked row takes the masked path for all its rows (it is exact for
        // unmasked rows too).
        float mt;
        if (__all_sync(0xffffffffu, hl >= kBN - 1)) {
          const float mx0 = i80 ? half_max<true, false>(sv, 0, 0, c0)
                                : half_max<false, false>(sv, 0, 0, c0);
          const float mx1 = i81 ? half_max<true, false>(sv, kHalf, 0, c1)
                                : half_max<false, false>(sv, kHalf, 0, c1);
          mt = fmaxf(mx0, mx1);
        } else {
          mt = masked_row_max(lane_addr, i80, i81, c0, c1, hl);
        }
        // Lazy rescaling: keep the old max unless the tile exceeds it by more
        // than 2^threshold, so P <= 2^threshold stays in fp16 range.
        const bool need = mt > m_run + kRescaleThreshold;
        if (n > 0 && __any_sync(0xffffffffu, need)) {
          // S_t(n) is ready, so P V_t(n-1) completed (the MMA thread issues
          // Q K^T_t(n) after it): O_t can be rescaled now.
          rescale_o<D>(lane_addr + C::kOCol, need ? ex2_approx(m_run - mt) : 1.0f);
        }
        if (need) {
          l_run *= ex2_approx(m_run - mt);  // 0 while m_run is -inf
          m_run = mt;
        }
        // Rows with no legal key yet keep m = -inf: their P is 0 (2^-inf).
        const float m_eff = m_run == -CUDART_INF_F ? 0.0f : m_run;
        // INT8 KV cache: P f = 2^(S c - m + log2 f) goes to the P V product
        // (<= 2^9, fp16-safe); the row sum divides f out again.
        const float me0 = KV8 ? m_eff - __log2f(fv0) : m_eff;
        const float me1 = KV8 ? m_eff - __log2f(fv1) : m_eff;
        // P, 32 keys at a time (the scores come from TMEM again: one copy of
        // each chunk's code stays hot in the instruction cache)
        // the row sum of this tile (with the INT8 cache: P f / f)
        float lsum = 0.0f;
        const float rf0 = KV8 ? 1.0f / fv0 : 1.0f, rf1 = KV8 ? 1.0f / fv1 : 1.0f;
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          const bool h1 = q >= 2;
          const bool i8 = h1 ? i81 : i80;
          const float cc = h1 ? c1 : c0;
          const float mm = h1 ? me1 : me0;
          const int hq = hl - 32 * q;
          float cs;
          if (__all_sync(0xffffffffu, hq >= 31)) {  // warp-uniform, as above
            uint32_t s32[32], pk[16];
            tmem_ld32(lane_addr + 32 * q, s32);
            tmem_ld_wait();
            float2 sa = make_float2(0.f, 0.f), sb = sa;
            if (i8) chunk_exp<true, false>(s32, cc, mm, 0, pk, sa, sb);
            else chunk_exp<false, false>(s32, cc, mm, 0, pk, sa, sb);
            tmem_st16(lane_addr + 16 * q, pk);
            const float2 cs2 = __fadd2_rn(sa, sb);
            cs = cs2.x + cs2.y;
          } else {
            cs = masked_chunk_exp(lane_addr + 32 * q, lane_addr + 16 * q, i8, cc,
                                  mm, hq);
          }
          lsum += cs * (h1 ? rf1 : rf0);
        }
        l_run += lsum;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[C::kBarP + t]);
      }

      // Epilogue: O / l.
      if (ok) {
        const bool got_last = mbar_wait(&bars[C::kBarO + t], 0, abort_flag);
        ok = __all_sync(0xffffffffu, got_last);
      }
      if (ok) {
        tc_fence_after();
        const bool valid = r_local < len;
        const float inv_l = 1.0f / l_run;
        // A tile whose 128 rows all lie in the sequence leaves through one
        // bulk store from shared memory (its Q buffer is free now); a
        // partial tile stores its valid rows directly.
        const bool full = row_base + t * kBM + kBM <= len;
        uint8_t* stage = sQ(t);
        uint16_t* orow =
            p.out + (static_cast<size_t>(start + r_local) * p.hq + h) * D;
#pragma unroll
        for (int oc = 0; oc < D; oc += 32) {
          uint32_t o[32];
          tmem_ld32(lane_addr + C::kOCol + oc, o);
          tmem_ld_wait();
          uint32_t hv[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            hv[j] = pack_half2(__uint_as_float(o[2 * j]) * inv_l,
                               __uint_as_float(o[2 * j + 1]) * inv_l);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 val = make_uint4(hv[4 * v], hv[4 * v + 1], hv[4 * v + 2],
                                         hv[4 * v + 3]);
            if (full) {
              // column oc + 8v: chunk oc / 64, 16-byte unit (oc % 64) / 8 + v
              // of row r, 128B swizzle
              const int col = oc + 8 * v;
              const uint32_t off = (col / 64) * (kBM * 128) + r * 128 +
                                   ((col % 64) / 8) * 16;
              *reinterpret_cast<uint4*>(stage + swz(off, 7)) = val;
            } else if (valid) {
              reinterpret_cast<uint4*>(orow + oc)[v] = val;
            }
          }
        }
        if (full) {
          fence_proxy_async_smem();  // staged O visible to the bulk copy
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[C::kBarOStage + t]);
          if (r == 0) {
            if (mbar_wait(&bars[C::kBarOStage + t], 0, abort_flag)) {
              for (int c = 0; c < D / 64; ++c)
                tma_store_3d(&p.tm_o, stage + c * kBM * 128, c * 64,
                             start + row_base + t * kBM, h);
              bulk_commit_group();
              bulk_wait_all();
            } else {
              ok = false;
            }
          }
        }
        if (p.lse && valid)
          p.lse[static_cast<size_t>(h) * p.total_tokens + start + r_local] =
              (m_run + __log2f(l_run)) * 0.69314718055994530942f;
      }
    }
    if (!ok) fail();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) tmem_dealloc(tmem, 512);
}

template <int D, bool KV8>
cudaError_t launch_rows_one(const AttnParams& p, cudaStream_t stream) {
  using C = RowCfg<D, KV8>;
  auto kern = attn_rows_kernel<D, KV8>;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const int pairs = (p.max_seqlen + 2 * kBM - 1) / (2 * kBM);
  dim3 grid(p.hq, pairs, p.batch);
  kern<<<grid, kThreads, C::kSmem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_rows(const AttnParams& p, int head_dim, bool kv8,
                             cudaStream_t stream) {
  if (head_dim == 128)
    return kv8 ? launch_rows_one<128, true>(p, stream)
               : launch_rows_one<128, false>(p, stream);
  if (head_dim == 64)
    return kv8 ? launch_rows_one<64, true>(p, stream)
               : launch_rows_one<64, false>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace tilemix
