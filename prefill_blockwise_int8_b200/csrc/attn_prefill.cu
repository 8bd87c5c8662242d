// Fused causal tile-routed FP16/INT8 prefill attention for sm_100a.
//
// Method: TileMix (arXiv 2608.17336).  Section 3 Preliminaries of the
// paperlayer summary: scores S = QK^T, online softmax keeping row maxima and
// normalisers, one 64-bit routing word per query-tile row whose bit
// floor(n/g) picks INT8 (Q8 K8^T, INT32 accumulation, rescaled by the block
// scales) or FP16 for key tile n; legality (causal, sequence end) decided
// separately from routing (appendix B).  Both paths update one shared
// online-softmax state and the FP16 P V product (ainews summary; appendix C).
//
// B200 design.  A CTA owns kQT 128-row query tiles of one head of one
// sequence (two tiles, rows 256M .. 256M+255; one tile with 64-row routing
// words) and walks the 128-key compute tiles of their causal range:
//   warp 8      TMA producer: Q and/or Q8 of its query tiles once, then per
//               key tile the K tile in every format a query tile routes some
//               of it to (fp16 and/or int8) and the fp16 V tile;
//   warp 9      one thread issues tcgen05.mma: S_t = Q_t K^T (kind::f16, f32
//               in TMEM) or Q8_t K8^T (kind::i8, s32 in TMEM) per 64-key half
//               of the tile (one N = 128 instruction chain when both halves
//               take the same path), and O_t += P_t V with P_t read from TMEM
//               (kind::f16, f32 TMEM accumulator);
//   warps 0-7   softmax: with two query tiles, warps 0-3 serve tile 0 and
//               warps 4-7 tile 1 (one thread per score row = TMEM lane), and
//               the two warpgroups interleave on every SM sub-partition; with
//               one query tile warps 0-3 take keys 0..63 and warps 4-7 keys
//               64..127 of each row and combine row max and sum through
//               shared memory.  Per tile: INT32 scores rescaled by
//               q_scale * k_scale, causal / end-of-sequence masking, running
//               max and sum in fp32, lazy rescale of O in TMEM when the max
//               grows by more than 2^8, P back to TMEM as fp16; then O / l.
// 128-key tiles keep every FP16 MMA at N = 128: on sm_100a a kind::f16
// M128 K16 instruction costs about the same at N = 64 as at N = 128.
#include <cuda.h>
#include <cuda_fp16.h>
#include <climits>
#include <math_constants.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace tilemix {
namespace {

constexpr int kBM = 128;     // query rows per tile = TMEM lanes = MMA M
constexpr int kBN = 128;     // keys per compute tile
constexpr int kHalf = 64;    // routing granularity inside a compute tile
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;
constexpr int kThreads = 320;
constexpr int kSmemBudget = 232448;  // max dynamic smem per block on sm_100
constexpr uint32_t kKindF16 = 1, kKindI8 = 2;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when the
                                           // row max grows by more than 2^8

__host__ __device__ constexpr int align1k(int x) { return (x + 1023) & ~1023; }

template <int D, bool DUAL>
struct Cfg {
  // DUAL (64-row routing words): a 128-row query tile may need both paths
  // for the same keys, so S has an fp16 and an int8 region and the CTA
  // holds one query tile.
  static constexpr int kQT = DUAL ? 1 : 2;
  static constexpr int kQBytes = kBM * D * 2;   // per query tile
  static constexpr int kQ8Bytes = kBM * D;
  static constexpr int kK16Bytes = kBN * D * 2;
  static constexpr int kK8Bytes = kBN * D;
  static constexpr int kVBytes = kBN * D * 2;
  static constexpr int kQ8Off = kQT * kQBytes;
  static constexpr int kRing0 = align1k(kQ8Off + kQT * kQ8Bytes);
  static constexpr int kK8Off = align1k(kK16Bytes);
  static constexpr int kKSlotBytes = align1k(kK8Off + kK8Bytes);
  static constexpr int kVSlotBytes = align1k(kVBytes);
  static constexpr int kRedBytes = DUAL ? 4096 : 0;  // row max / sum exchange
  static constexpr int kBarBytes = 512;
  static constexpr int kAvail =
      kSmemBudget - 1024 - kBarBytes - kRedBytes - kRing0;
  // Two V slots (P V of every query tile must finish before a V slot
  // frees), then as many K slots as fit (at most 3).
  static constexpr int kVStages = 2;
  static constexpr int kKFit = (kAvail - kVStages * kVSlotBytes) / kKSlotBytes;
  static constexpr int kKStages = kKFit > 3 ? 3 : kKFit;
  static_assert(kKStages >= 1, "shared memory too small");
  static constexpr int kVRing0 = kRing0 + kKStages * kKSlotBytes;
  static constexpr int kRedOff = kVRing0 + kVStages * kVSlotBytes;
  static constexpr int kBarOff = kRedOff + kRedBytes;
  static constexpr int kSmem = kBarOff + kBarBytes + 1024;  // + align slack
  static_assert(kSmem - 1024 <= kSmemBudget, "shared memory overflow");
  // TMEM columns of query tile t start at t * kTileCols: the S region(s),
  // then O (D columns).
  static constexpr int kS16 = 0;
  static constexpr int kS8 = DUAL ? kBN : 0;
  static constexpr int kOCol = DUAL ? 2 * kBN : kBN;
  // P (fp16 pairs, 64 columns): over the consumed S columns with two query
  // tiles; in spare columns with one, where the two warpgroups read the
  // fp16 S region while the other may already store P.
  static constexpr int kP = DUAL ? 3 * kBN : 0;
  static constexpr int kTileCols = DUAL ? 512 : 256;
  static constexpr int kTmemCols = 512;
  static_assert(kOCol + D <= kTileCols, "TMEM overflow");
  // barrier indices
  static constexpr int kBarQ = 0;
  static constexpr int kBarK = 1;
  static constexpr int kBarKEmpty = kBarK + kKStages;
  static constexpr int kBarV = kBarKEmpty + kKStages;
  static constexpr int kBarVEmpty = kBarV + kVStages;
  static constexpr int kBarS = kBarVEmpty + kVStages;  // [tile]
  static constexpr int kBarP = kBarS + 2;              // [tile]
  static constexpr int kBarO = kBarP + 2;              // [tile]
  static constexpr int kBarRed = kBarO + 2;            // one tile: [2]
  static constexpr int kBarDrain = kBarRed + 2;
  static constexpr int kNumBars = kBarDrain + 1;
  static_assert(kNumBars * 8 + 16 <= kBarBytes, "barrier area");
};

// K-major fp16 operand stored as D/64 column chunks of [rows][128 B] with
// the 128-byte swizzle; `chunk_bytes` = rows * 128; ks = K-step of 16.
__device__ __forceinline__ uint64_t desc_k_f16(uint32_t base, int chunk_bytes,
                                               int ks) {
  const uint32_t addr = base + (ks >> 2) * chunk_bytes + (ks & 3) * 32;
  return smem_desc(addr, 16, 1024, kSwizzle128);
}

// K-major int8 operand (rows x D bytes); ks = K-step of 32 bytes.
template <int D>
__device__ __forceinline__ uint64_t desc_k_i8(uint32_t base, int ks) {
  return smem_desc(base + ks * 32, 16, 8 * D,
                   D == 128 ? kSwizzle128 : kSwizzle64);
}

// MN-major fp16 V tile (128 keys x D) stored as D/64 chunks [128][128 B];
// ks = K-step of 16 keys.  LBO = chunk stride, SBO = 8 keys.
__device__ __forceinline__ uint64_t desc_v(uint32_t base, int ks) {
  return smem_desc(base + ks * 16 * 128, kBN * 128, 1024, kSwizzle128);
}

// Routing state of one 128-row query tile.
struct TileRoute {
  uint64_t w0, w1;  // words of rows 0..63 / 64..127 (equal unless DUAL)
  int nl0, nl1;     // last legal 64-key block of each row half (-1: none)
  int n_last;       // last legal 128-key tile (-1: no rows)
};

template <int D, bool DUAL>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  using C = Cfg<D, DUAL>;
  constexpr int kQT = C::kQT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Grid (head, query-tile group, sequence): all tiles of one sequence run
  // together so its K/V stays in L2; longest query tiles first inside it.
  const int h = blockIdx.x;
  const int mp = gridDim.y - 1 - blockIdx.y;
  const int b = blockIdx.z;

  // A status word that already holds an error (an earlier CTA timed out or
  // saw bad lengths) stops every later CTA before it does any work.
  if (p.status && *reinterpret_cast<volatile int32_t*>(p.status) != 0) return;

  // ---- per-CTA problem geometry (uniform across the CTA) ----
  const int start = p.cu_seqlens[b];
  const int len = p.cu_seqlens[b + 1] - start;
  if (start < 0 || len < 0 || len > p.max_seqlen ||
      start + len > p.total_tokens) {
    if (threadIdx.x == 0) report_status(p.status, kStatusBadSeqlens);
    return;
  }
  const int row_base = mp * (kQT * kBM);
  if (row_base >= len) return;
  const int hk = p.head_map ? p.head_map[h] : h / p.heads_per_kv;
  if (hk < 0 || hk >= p.hkv) {
    if (threadIdx.x == 0) report_status(p.status, kStatusBadSeqlens);
    return;
  }

  const bool routed = !p.fp16_only;  // the mask may be NULL otherwise
  const size_t wbase = (static_cast<size_t>(b) * p.hkv + hk) * p.tm_route;
  auto route_of = [&](int t) {
    const int row0 = row_base + t * kBM;
    TileRoute r{0ull, 0ull, -1, -1, -1};
    if (t < kQT && row0 < len) {
      const int last = min(row0 + kBM - 1, len - 1);
      r.n_last = last / kBN;
      if (DUAL) {
        const int rr = row0 / 64;
        r.w0 = routed ? p.mask[wbase + rr] : 0ull;
        r.nl0 = min(row0 + 63, len - 1) / kHalf;
        if (row0 + 64 < len) {
          r.w1 = routed ? p.mask[wbase + rr + 1] : 0ull;
          r.nl1 = last / kHalf;
        }
      } else {
        r.w0 = r.w1 = routed ? p.mask[wbase + row0 / kBM] : 0ull;
        r.nl0 = r.nl1 = last / kHalf;
      }
    }
    return r;
  };
  const TileRoute rt0 = route_of(0), rt1 = route_of(1);
  auto rt = [&](int t) -> const TileRoute& { return t ? rt1 : rt0; };
  const int n_end = max(rt0.n_last, rt1.n_last);
  const int tpb = p.tiles_per_bit;  // 64-key blocks per routing bit
  // Paths query tile t needs for 64-key half kh of key tile n (0: none).
  auto kinds_of = [&](int t, int n, int kh) -> uint32_t {
    const TileRoute& r = rt(t);
    const int n64 = 2 * n + kh;
    const int gi = n64 / tpb;
    uint32_t k = 0;
    if (n64 <= r.nl0) k |= ((r.w0 >> gi) & 1ull) ? kKindI8 : kKindF16;
    if (n64 <= r.nl1) k |= ((r.w1 >> gi) & 1ull) ? kKindI8 : kKindF16;
    return k;
  };

  // ---- shared memory carve-up ----
  auto sQ = [&](int t) { return smem + t * C::kQBytes; };
  auto sQ8 = [&](int t) { return smem + C::kQ8Off + t * C::kQ8Bytes; };
  auto kslot = [&](int s) { return smem + C::kRing0 + s * C::kKSlotBytes; };
  auto vslot = [&](int s) { return smem + C::kVRing0 + s * C::kVSlotBytes; };
  // one query tile: [max | sum][tile parity][warpgroup][row]
  float* red = reinterpret_cast<float*>(smem + C::kRedOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (warp == kWarpProducer && lane == 0) {
    mbar_init(&bars[C::kBarQ], 1);
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(&bars[C::kBarK + s], 1);
      mbar_init(&bars[C::kBarKEmpty + s], 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(&bars[C::kBarV + s], 1);
      mbar_init(&bars[C::kBarVEmpty + s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[C::kBarS + i], 1);
      mbar_init(&bars[C::kBarP + i], DUAL ? 256 : 128);
      mbar_init(&bars[C::kBarO + i], 1);
      mbar_init(&bars[C::kBarRed + i], 256);
    }
    mbar_init(&bars[C::kBarDrain], 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
    if (routed) {  // the INT8 maps are left empty in FP16-only mode
      tma_prefetch_desc(&p.tm_q8);
      tma_prefetch_desc(&p.tm_k8);
    }
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, C::kTmemCols);
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

  if (warp == kWarpProducer) {
    // =================== TMA producer ===================
    if (lane == 0) {
      uint32_t qbytes = 0;
      uint32_t need[2] = {0u, 0u};
      for (int t = 0; t < kQT; ++t) {
        for (int n = 0; n <= rt(t).n_last; ++n)
          need[t] |= kinds_of(t, n, 0) | kinds_of(t, n, 1);
        qbytes += ((need[t] & kKindF16) ? C::kQBytes : 0) +
                  ((need[t] & kKindI8) ? C::kQ8Bytes : 0);
      }
      mbar_arrive_expect_tx(&bars[C::kBarQ], qbytes);
      for (int t = 0; t < kQT; ++t) {
        const int qrow = start + row_base + t * kBM;
        if (need[t] & kKindF16)
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sQ(t) + c * kBM * 128, &p.tm_q, &bars[C::kBarQ],
                        c * 64, qrow, h);
        if (need[t] & kKindI8)
          tma_load_3d(sQ8(t), &p.tm_q8, &bars[C::kBarQ], 0, qrow, h);
      }
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      for (int n = 0; n <= n_end && ok; ++n) {
        const int krow = start + n * kBN;
        // K tile n in every format some query tile routes part of it to
        const int ks = n % C::kKStages;
        const int jk = n / C::kKStages;
        if (jk > 0 &&
            !mbar_wait(&bars[C::kBarKEmpty + ks], (jk - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        uint32_t kinds = 0;
        for (int t = 0; t < kQT; ++t)
          kinds |= kinds_of(t, n, 0) | kinds_of(t, n, 1);
        mbar_arrive_expect_tx(&bars[C::kBarK + ks],
                              ((kinds & kKindF16) ? C::kK16Bytes : 0) +
                                  ((kinds & kKindI8) ? C::kK8Bytes : 0));
        if (kinds & kKindF16)
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(kslot(ks) + c * kBN * 128, &p.tm_k,
                        &bars[C::kBarK + ks], c * 64, krow, hk);
        if (kinds & kKindI8)
          tma_load_3d(kslot(ks) + C::kK8Off, &p.tm_k8, &bars[C::kBarK + ks], 0,
                      krow, hk);
        k_issued = n + 1;
        // V tile n
        const int vs = n % C::kVStages;
        const int jv = n / C::kVStages;
        if (jv > 0 &&
            !mbar_wait(&bars[C::kBarVEmpty + vs], (jv - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&bars[C::kBarV + vs], C::kVBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(vslot(vs) + c * kBN * 128, &p.tm_v, &bars[C::kBarV + vs],
                      c * 64, krow, hk);
        v_issued = n + 1;
      }
      if (!ok) {
        fail();
        // Let the copies already in flight land before the CTA exits.
        mbar_wait(&bars[C::kBarQ], 0, nullptr);
        for (int n = max(0, k_issued - C::kKStages); n < k_issued; ++n)
          mbar_wait(&bars[C::kBarK + n % C::kKStages], (n / C::kKStages) & 1,
                    nullptr);
        for (int n = max(0, v_issued - C::kVStages); n < v_issued; ++n)
          mbar_wait(&bars[C::kBarV + n % C::kVStages], (n / C::kVStages) & 1,
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

      // S_t(n) = Q_t K(n)^T, each 64-key half on the path(s) it routes to.
      auto issue_qk = [&](int t, int n) -> bool {
        if (n > rt(t).n_last) return true;
        const uint32_t k0 = kinds_of(t, n, 0);
        uint32_t k1 = kinds_of(t, n, 1);
        if (k1 == 0) k1 = k0;  // keys past every row: any path will do
        const int s = n % C::kKStages;
        if (!mbar_wait(&bars[C::kBarK + s], (n / C::kKStages) & 1, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t kb = smem_u32(kslot(s));
        const uint32_t tb = tmem + t * C::kTileCols;
        const uint32_t halves16 = ((k0 & kKindF16) ? 1u : 0u) |
                                  ((k1 & kKindF16) ? 2u : 0u);
        const uint32_t halves8 = ((k0 & kKindI8) ? 1u : 0u) |
                                 ((k1 & kKindI8) ? 2u : 0u);
        if (halves16) {
          const uint32_t q16 = smem_u32(sQ(t));
          const bool both = halves16 == 3u;
          const uint32_t hoff = (halves16 == 2u) ? 1u : 0u;  // second half
          const uint32_t d = tb + C::kS16 + hoff * kHalf;
          const uint32_t bk = kb + hoff * (kHalf * 128);  // row 64 of a chunk
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_f16_ss(d, desc_k_f16(q16, kBM * 128, ks),
                       desc_k_f16(bk, kBN * 128, ks),
                       both ? id16_full : id16_half, ks > 0 ? 1u : 0u);
        }
        if (halves8) {
          const uint32_t q8 = smem_u32(sQ8(t));
          const bool both = halves8 == 3u;
          const uint32_t hoff = (halves8 == 2u) ? 1u : 0u;
          const uint32_t d = tb + C::kS8 + hoff * kHalf;
          const uint32_t bk = kb + C::kK8Off + hoff * (kHalf * D);
#pragma unroll
          for (int ks = 0; ks < D / 32; ++ks)
            mma_i8_ss(d, desc_k_i8<D>(q8, ks), desc_k_i8<D>(bk, ks),
                      both ? id8_full : id8_half, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars[C::kBarS + t]);
        return true;
      };
      // O_t += P_t(n) V(n), P_t(n) read from TMEM.
      auto issue_pv = [&](int t, int n) -> bool {
        if (n > rt(t).n_last) return true;
        const int s = n % C::kVStages;
        if (!mbar_wait(&bars[C::kBarP + t], n & 1, abort_flag)) return false;
        if (!mbar_wait(&bars[C::kBarV + s], (n / C::kVStages) & 1, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t vb = smem_u32(vslot(s));
        const uint32_t tb = tmem + t * C::kTileCols;
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks)
          mma_f16_ts(tb + C::kOCol, tb + C::kP + ks * 8, desc_v(vb, ks),
                     idesc_pv, (n > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&bars[C::kBarO + t]);
        return true;
      };

      // S is single-buffered per query tile: Q K^T of tile n+1 follows the
      // P V that reads P of tile n.  A K slot frees when every query tile's
      // Q K^T of it completed, a V slot when every P V did.
      for (int t = 0; t < kQT && ok; ++t) ok = issue_qk(t, 0);
      if (ok) mma_commit(&bars[C::kBarKEmpty + 0]);
      for (int n = 0; n <= n_end && ok; ++n) {
        for (int t = 0; t < kQT && ok; ++t) {
          ok = issue_pv(t, n);
          if (ok) ok = issue_qk(t, n + 1);
        }
        if (ok) {
          mma_commit(&bars[C::kBarVEmpty + n % C::kVStages]);
          if (n + 1 <= n_end)
            mma_commit(&bars[C::kBarKEmpty + (n + 1) % C::kKStages]);
        }
      }
      if (!ok) fail();
      // Drain: every MMA issued above has finished once this completes.
      mma_commit(&bars[C::kBarDrain]);
      mbar_wait(&bars[C::kBarDrain], 0, nullptr);
    }
    __syncwarp();
  } else {
    // =================== softmax warps 0-7 ===================
    // Two query tiles: warpgroup wg serves tile wg, all 128 keys of a tile.
    // One query tile (DUAL): warpgroup wg serves keys 64*wg .. 64*wg+63.
    const int wg = warp >> 2;
    const int t = DUAL ? 0 : wg;
    const int r = threadIdx.x & 127;  // score row = TMEM lane
    constexpr int kCols = DUAL ? kHalf : kBN;  // score columns per thread
    const int c0 = DUAL ? wg * kHalf : 0;      // first column of this thread
    const TileRoute R = rt(t);
    if (R.n_last >= 0) {
      const int r_local = row_base + t * kBM + r;
      const bool valid = r_local < len;
      const int rh = DUAL ? (r >> 6) : 0;  // routing row half
      const uint64_t my_w = rh ? R.w1 : R.w0;
      const int my_nl = rh ? R.nl1 : R.nl0;
      const uint32_t tb = tmem + t * C::kTileCols;
      const uint32_t lane_addr =
          tb + (static_cast<uint32_t>((warp & 3) * 32) << 16);
      const int key_lim = min(r_local, len - 1);  // keys j <= key_lim legal
      float sq = 0.0f;
      if (routed)
        sq = p.q_scale[(static_cast<size_t>(h) * p.batch + b) * p.nbq +
                       key_lim / p.quant_block_q];
      const float* kscale =
          routed ? p.k_scale + (static_cast<size_t>(hk) * p.batch + b) * p.nbk
                 : nullptr;
      // K scales of the next tile are fetched while this one is processed.
      auto ksc = [&](int n, int kh) {
        const int blk = (n * kBN + kh * kHalf) / p.quant_block_k;
        return kscale[min(blk, p.nbk - 1)];
      };
      float sk0_next = 0.f, sk1_next = 0.f;
      if (routed) {
        sk0_next = ksc(0, 0);
        sk1_next = ksc(0, 1);
      }

      float m_run = -CUDART_INF_F;
      float l_run = 0.0f;
      bool ok = true;
      for (int n = 0; n <= R.n_last; ++n) {
        const float sk0 = sk0_next, sk1 = sk1_next;
        if (routed && n < R.n_last) {
          sk0_next = ksc(n + 1, 0);
          sk1_next = ksc(n + 1, 1);
        }
        // Exits stay warp-uniform: the tcgen05.ld/st below are .sync.aligned.
        const bool got_s = mbar_wait(&bars[C::kBarS + t], n & 1, abort_flag);
        if (!__all_sync(0xffffffffu, got_s)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // Path of each 64-key half of this thread's columns for this row
        // (its routing row half).  kLH local halves, global half c0/64 + hh.
        constexpr int kLH = kCols / kHalf;
        bool i8l[kLH];
        float csl[kLH];
#pragma unroll
        for (int hh = 0; hh < kLH; ++hh) {
          const int n64 = 2 * n + c0 / kHalf + hh;
          i8l[hh] = (n64 <= my_nl) && (((my_w >> (n64 / tpb)) & 1ull) != 0);
        }
        // Keys past every row of the tile: the MMA wrote the other half's
        // path there; those values are masked below either way.
        if (!DUAL && 2 * n + 1 > my_nl) i8l[kLH - 1] = i8l[0];
#pragma unroll
        for (int hh = 0; hh < kLH; ++hh)
          csl[hh] = i8l[hh] ? p.scale_log2 * sq *
                                  ((c0 / kHalf + hh) ? sk1 : sk0)
                            : p.scale_log2;
        const int lim = key_lim - n * kBN - c0;  // columns j <= lim are legal
        const bool full = lim >= kCols - 1;
        auto s_col = [&](int hh) {
          return lane_addr + (i8l[hh] ? C::kS8 : C::kS16) + c0 + hh * kHalf;
        };

        // Pass 1: row max, 64 columns at a time (the scores stay in TMEM).
        // INT8 halves take the integer max of the raw accumulators.
        float m_tile = -CUDART_INF_F;
#pragma unroll
        for (int hh = 0; hh < kLH; ++hh) {
          uint32_t sv[kHalf];
          tmem_ld32(s_col(hh), *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
          tmem_ld32(s_col(hh) + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
          tmem_ld_wait();
          const int hl = lim - hh * kHalf;  // legal columns of this half: <= hl
          if (p.qk_dump && valid && i8l[hh] && 2 * n + c0 / kHalf + hh <= my_nl) {
            const int n64 = 2 * n + c0 / kHalf + hh;
            const int rrow = r_local / p.route_bm;
            const int rr = r_local - rrow * p.route_bm;
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
            const int keys_left = len - key0;  // keys inside the sequence
#pragma unroll
            for (int j = 0; j < kHalf; ++j)
              if (j < keys_left) dst[j] = static_cast<int32_t>(sv[j]);
          }
          float mx;
          if (i8l[hh]) {
            int a0 = INT_MIN, a1 = INT_MIN, a2 = INT_MIN, a3 = INT_MIN;
#pragma unroll
            for (int j = 0; j < kHalf; j += 4) {
              const bool fullh = hl >= kHalf - 1;
              a0 = max(a0, (fullh || j <= hl) ? static_cast<int>(sv[j]) : INT_MIN);
              a1 = max(a1, (fullh || j + 1 <= hl) ? static_cast<int>(sv[j + 1]) : INT_MIN);
              a2 = max(a2, (fullh || j + 2 <= hl) ? static_cast<int>(sv[j + 2]) : INT_MIN);
              a3 = max(a3, (fullh || j + 3 <= hl) ? static_cast<int>(sv[j + 3]) : INT_MIN);
            }
            const int im = max(max(a0, a1), max(a2, a3));
            mx = (hl < 0) ? -CUDART_INF_F : static_cast<float>(im);
          } else {
            float a0 = -CUDART_INF_F, a1 = -CUDART_INF_F, a2 = -CUDART_INF_F,
                  a3 = -CUDART_INF_F;
            auto g = [&](int j) {
              return (hl >= kHalf - 1 || j <= hl) ? __uint_as_float(sv[j])
                                                  : -CUDART_INF_F;
            };
#pragma unroll
            for (int j = 0; j < kHalf; j += 8) {
              a0 = fmax3(a0, g(j), g(j + 1));
              a1 = fmax3(a1, g(j + 2), g(j + 3));
              a2 = fmax3(a2, g(j + 4), g(j + 5));
              a3 = fmax3(a3, g(j + 6), g(j + 7));
            }
            mx = fmax3(a0, a1, fmaxf(a2, a3));
          }
          if (mx != -CUDART_INF_F) m_tile = fmaxf(m_tile, mx * csl[hh]);
        }
        if (DUAL) {
          // the two warpgroups hold the two halves of each row
          red[(n & 1) * 256 + wg * 128 + r] = m_tile;
          mbar_arrive(&bars[C::kBarRed + (n & 1)]);
          const bool got_r =
              mbar_wait(&bars[C::kBarRed + (n & 1)], (n >> 1) & 1, abort_flag);
          if (!__all_sync(0xffffffffu, got_r)) {
            ok = false;
            break;
          }
          m_tile = fmaxf(m_tile, red[(n & 1) * 256 + (1 - wg) * 128 + r]);
        }
        const float m_new = fmaxf(m_run, m_tile);
        const bool need = m_new > m_run + kRescaleThreshold;

        if (n > 0) {
          // O holds P V of every tile before n once PV(n-1) completed.
          const bool got_o =
              mbar_wait(&bars[C::kBarO + t], (n - 1) & 1, abort_flag);
          if (!__all_sync(0xffffffffu, got_o)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (__any_sync(0xffffffffu, need)) {
            const float alpha = need ? ex2_approx(m_run - m_new) : 1.0f;
            // with one query tile each warpgroup rescales half of O
            constexpr int kOCols = DUAL ? D / 2 : D;
            const int o0 = DUAL ? wg * (D / 2) : 0;
#pragma unroll
            for (int oc = 0; oc < kOCols; oc += 32) {
              uint32_t o[32];
              tmem_ld32(lane_addr + C::kOCol + o0 + oc, o);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j)
                o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
              tmem_st32(lane_addr + C::kOCol + o0 + oc, o);
            }
          }
        }
        if (need) {
          l_run *= ex2_approx(m_run - m_new);
          m_run = m_new;
        }
        // Pass 2: P = 2^(x - m) as fp16 pairs, key 2i of this thread's
        // columns in the low half of P column (c0 / 2 + i); packed partial
        // sums.  INT32 accumulators convert to fp32 exactly (|acc| <= 127^2 d
        // < 2^22) on the integer and FMA pipes, not the conversion unit.
        float2 ps0 = make_float2(0.f, 0.f), ps1 = ps0, ps2 = ps0, ps3 = ps0;
        const float2 nm2 = make_float2(-m_run, -m_run);
#pragma unroll
        for (int hh = 0; hh < kLH; ++hh) {
          uint32_t sv[kHalf];
          tmem_ld32(s_col(hh), *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
          tmem_ld32(s_col(hh) + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
          tmem_ld_wait();
          if (i8l[hh]) {
#pragma unroll
            for (int j = 0; j < kHalf; j += 2) {
              const float2 biased =
                  make_float2(__uint_as_float(sv[j] + kIntBiasBits),
                              __uint_as_float(sv[j + 1] + kIntBiasBits));
              const float2 v =
                  __fadd2_rn(biased, make_float2(-kIntBias, -kIntBias));
              sv[j] = __float_as_uint(v.x);
              sv[j + 1] = __float_as_uint(v.y);
            }
          }
          const float2 c2 = make_float2(csl[hh], csl[hh]);
          const int hl = lim - hh * kHalf;
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int j = 2 * i;
            const float2 x = __ffma2_rn(
                make_float2(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])),
                c2, nm2);
            float2 pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            if (!full) {  // masked keys: exactly 0
              pr.x = (j <= hl) ? pr.x : 0.0f;
              pr.y = (j + 1 <= hl) ? pr.y : 0.0f;
            }
            switch (i & 3) {
              case 0: ps0 = __fadd2_rn(ps0, pr); break;
              case 1: ps1 = __fadd2_rn(ps1, pr); break;
              case 2: ps2 = __fadd2_rn(ps2, pr); break;
              default: ps3 = __fadd2_rn(ps3, pr); break;
            }
            pk[i] = pack_half2(pr.x, pr.y);
          }
          tmem_st32(lane_addr + C::kP + (c0 + hh * kHalf) / 2, pk);
        }
        const float2 s4 = __fadd2_rn(__fadd2_rn(ps0, ps1), __fadd2_rn(ps2, ps3));
        float lsum = s4.x + s4.y;
        if (DUAL) red[512 + (n & 1) * 256 + wg * 128 + r] = lsum;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars[C::kBarP + t]);
        if (DUAL) {
          // both halves' sums are in shared memory once the P barrier
          // (both warpgroups' arrivals) completes
          const bool got_p = mbar_wait(&bars[C::kBarP + t], n & 1, abort_flag);
          if (!__all_sync(0xffffffffu, got_p)) {
            ok = false;
            break;
          }
          lsum += red[512 + (n & 1) * 256 + (1 - wg) * 128 + r];
        }
        l_run += lsum;
      }

      const bool got_last =
          ok && mbar_wait(&bars[C::kBarO + t], R.n_last & 1, abort_flag);
      if (__all_sync(0xffffffffu, got_last)) {
        tc_fence_after();
        const float inv_l = 1.0f / l_run;
        constexpr int kOCols = DUAL ? D / 2 : D;
        const int o0 = DUAL ? wg * (D / 2) : 0;
        uint16_t* orow =
            p.out + (static_cast<size_t>(start + r_local) * p.hq + h) * D + o0;
#pragma unroll
        for (int oc = 0; oc < kOCols; oc += 32) {
          uint32_t o[32];
          tmem_ld32(lane_addr + C::kOCol + o0 + oc, o);
          tmem_ld_wait();
          uint32_t hv[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            hv[j] = pack_half2(__uint_as_float(o[2 * j]) * inv_l,
                               __uint_as_float(o[2 * j + 1]) * inv_l);
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + oc);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(hv[4 * v], hv[4 * v + 1], hv[4 * v + 2],
                                  hv[4 * v + 3]);
          }
        }
        if (p.lse && valid && wg == t)
          p.lse[static_cast<size_t>(h) * p.total_tokens + start + r_local] =
              (m_run + __log2f(l_run)) * 0.69314718055994530942f;
      } else {
        fail();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) tmem_dealloc(tmem, C::kTmemCols);
}

template <int D, bool DUAL>
cudaError_t launch_one(const AttnParams& p, cudaStream_t stream) {
  using C = Cfg<D, DUAL>;
  auto kern = attn_fwd_kernel<D, DUAL>;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const int groups = (p.max_seqlen + C::kQT * kBM - 1) / (C::kQT * kBM);
  dim3 grid(p.hq, groups, p.batch);
  kern<<<grid, kThreads, C::kSmem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_prefill(const AttnParams& p, const AttnLaunchShape& s,
                                cudaStream_t stream) {
  if (s.head_dim == 128)
    return s.dual ? launch_one<128, true>(p, stream)
                  : launch_one<128, false>(p, stream);
  if (s.head_dim == 64)
    return s.dual ? launch_one<64, true>(p, stream)
                  : launch_one<64, false>(p, stream);
  return cudaErrorInvalidValue;
}

int attn_smem_bytes(const AttnLaunchShape& s) {
  if (s.head_dim == 128)
    return s.dual ? Cfg<128, true>::kSmem : Cfg<128, false>::kSmem;
  if (s.head_dim == 64)
    return s.dual ? Cfg<64, true>::kSmem : Cfg<64, false>::kSmem;
  return -1;
}

}  // namespace tilemix
