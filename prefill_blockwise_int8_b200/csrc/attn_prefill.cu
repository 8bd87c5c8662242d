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
// B200 design.  One CTA = two 128-row query tiles (rows 256M .. 256M+255 of
// one head of one sequence) sharing every K/V tile it loads:
//   warp 8      TMA producer: Q / Q8 of both tiles once, then per 64-key tile
//               the K tile in every format a query tile routes it to (fp16
//               and/or int8) and the fp16 V tile, into a ring of stages;
//   warp 9      one thread issues tcgen05.mma: S_t = Q_t K^T (kind::f16, f32
//               in TMEM) or S_t = Q8_t K8^T (kind::i8, s32 in TMEM), and
//               O_t += P_t V with P_t read from TMEM (kind::f16, f32 TMEM
//               accumulator); Q K^T runs two key tiles ahead of P V (S is
//               double-buffered per query tile);
//   warps 0-3   softmax warpgroup of query tile 0, warps 4-7 of tile 1; a
//               thread owns one score row (TMEM lane): rescale of INT32 scores
//               by q_scale * k_scale, causal / end-of-sequence masking,
//               running max and sum in fp32, lazy rescale of O in TMEM when
//               the max grows by more than 2^8, P back to TMEM as fp16, and
//               the final O / l epilogue.
// The two softmax warpgroups interleave on every SM sub-partition, so one's
// exponentials overlap the other's TMEM loads, reductions and barriers.
//
// Score tiles are 128 x 64 on the tensor cores; a routing tile of 128 keys is
// two compute tiles that read the same bit.  With 64-row routing words
// (block_m = 64) a 128-row query tile covers two routing rows; a key tile
// whose two halves route differently is computed on both paths into separate
// TMEM buffers (S single-buffered then) and each row reads its own.
#include <cuda.h>
#include <cuda_fp16.h>
#include <math_constants.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace tilemix {
namespace {

constexpr int kBM = 128;     // query rows per tile = TMEM lanes = MMA M
constexpr int kBN = 64;      // keys per compute tile
constexpr int kQT = 2;       // query tiles per CTA
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
  static constexpr int kQBytes = kBM * D * 2;   // per query tile
  static constexpr int kQ8Bytes = kBM * D;
  static constexpr int kK16Bytes = kBN * D * 2;
  static constexpr int kK8Bytes = kBN * D;
  static constexpr int kVBytes = kBN * D * 2;
  static constexpr int kQ8Off = kQT * kQBytes;
  static constexpr int kRing0 = align1k(kQ8Off + kQT * kQ8Bytes);
  // Separate K and V rings: a K slot is free once both query tiles' Q K^T
  // read it, long before P V is done with the V tile of the same keys.  A K
  // slot holds both formats (the query tiles may route a key tile
  // differently).
  static constexpr int kK8Off = align1k(kK16Bytes);
  static constexpr int kKSlotBytes = align1k(kK8Off + kK8Bytes);
  static constexpr int kVSlotBytes = align1k(kVBytes);
  static constexpr int kBarBytes = 256;
  static constexpr int kStagesFit = (kSmemBudget - 1024 - kBarBytes - kRing0) /
                                    (kKSlotBytes + kVSlotBytes);
  static constexpr int kStages = kStagesFit > 4 ? 4 : kStagesFit;
  static_assert(kStages >= 3, "shared memory too small for three stages");
  static constexpr int kVRing0 = kRing0 + kStages * kKSlotBytes;
  static constexpr int kBarOff = kVRing0 + kStages * kVSlotBytes;
  static constexpr int kSmem = kBarOff + kBarBytes + 1024;  // + align slack
  // TMEM: 256 columns per query tile.  S slots of 64 columns (f32 / s32)
  // at [0, 128), O (D columns) at 128.
  static constexpr int kSlots = DUAL ? 1 : 2;  // S buffers per query tile
  static constexpr int kTileCols = 256;
  static constexpr int kOCol = 128;
  static constexpr int kTmemCols = 512;
  static_assert(D <= 128, "O must fit in 128 TMEM columns");
  static constexpr int s16_col(int slot) { return DUAL ? 0 : slot * kBN; }
  static constexpr int s8_col(int slot) { return DUAL ? kBN : slot * kBN; }
  // barrier indices
  static constexpr int kBarQ = 0;
  static constexpr int kBarK = 1;
  static constexpr int kBarKEmpty = kBarK + kStages;
  static constexpr int kBarV = kBarKEmpty + kStages;
  static constexpr int kBarVEmpty = kBarV + kStages;
  static constexpr int kBarS = kBarVEmpty + kStages;    // [tile][slot]
  static constexpr int kBarP = kBarS + kQT * 2;         // [tile][slot]
  static constexpr int kBarO = kBarP + kQT * 2;         // [tile]
  static constexpr int kBarDrain = kBarO + kQT;
  static constexpr int kNumBars = kBarDrain + 1;
  static_assert(kNumBars * 8 + 16 <= kBarBytes, "barrier area");
};

// K-major fp16 operand (rows x D) stored as D/64 column chunks, each
// [rows][128 B] with the 128-byte swizzle; ks = K-step of 16 elements.
__device__ __forceinline__ uint64_t desc_k_f16(uint32_t base, int rows, int ks) {
  const uint32_t addr = base + (ks >> 2) * (rows * 128) + (ks & 3) * 32;
  return smem_desc(addr, 16, 1024, kSwizzle128);
}

// K-major int8 operand (rows x D bytes); ks = K-step of 32 bytes.
template <int D>
__device__ __forceinline__ uint64_t desc_k_i8(uint32_t base, int ks) {
  return smem_desc(base + ks * 32, 16, 8 * D,
                   D == 128 ? kSwizzle128 : kSwizzle64);
}

// MN-major fp16 V tile (64 keys x D) stored as D/64 chunks [64][128 B];
// ks = K-step of 16 keys.  LBO = chunk stride, SBO = 8 keys.
__device__ __forceinline__ uint64_t desc_v(uint32_t base, int ks) {
  return smem_desc(base + ks * 16 * 128, kBN * 128, 1024, kSwizzle128);
}

// Routing state of one 128-row query tile.
struct TileRoute {
  uint64_t w0, w1;  // words of rows 0..63 / 64..127 (equal unless DUAL)
  int nl0, nl1;     // last legal 64-key tile of each half (-1: no rows)
  int n_last;       // last legal 64-key tile of the tile (-1: no tile)
};

template <int D, bool DUAL>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  using C = Cfg<D, DUAL>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Grid (head, query-tile pair, sequence): all tiles of one sequence run
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
    if (row0 < len) {
      r.n_last = min(row0 + kBM - 1, len - 1) / kBN;
      if (DUAL) {
        const int rr = row0 / 64;
        r.w0 = routed ? p.mask[wbase + rr] : 0ull;
        r.nl0 = min(row0 + 63, len - 1) / kBN;
        if (row0 + 64 < len) {
          r.w1 = routed ? p.mask[wbase + rr + 1] : 0ull;
          r.nl1 = r.n_last;
        }
      } else {
        r.w0 = r.w1 = routed ? p.mask[wbase + row0 / kBM] : 0ull;
        r.nl0 = r.nl1 = r.n_last;
      }
    }
    return r;
  };
  const TileRoute rt0 = route_of(0), rt1 = route_of(1);
  auto rt = [&](int t) -> const TileRoute& { return t ? rt1 : rt0; };
  const int n_end = max(rt0.n_last, rt1.n_last);
  const int tpb = p.tiles_per_bit;
  // Which score paths query tile t needs for key tile n (0: not legal).
  auto kinds_of = [&](int t, int n) -> uint32_t {
    const TileRoute& r = rt(t);
    const int gi = n / tpb;
    uint32_t k = 0;
    if (n <= r.nl0) k |= ((r.w0 >> gi) & 1ull) ? kKindI8 : kKindF16;
    if (n <= r.nl1) k |= ((r.w1 >> gi) & 1ull) ? kKindI8 : kKindF16;
    return k;
  };

  // ---- shared memory carve-up ----
  auto sQ = [&](int t) { return smem + t * C::kQBytes; };
  auto sQ8 = [&](int t) { return smem + C::kQ8Off + t * C::kQ8Bytes; };
  auto kslot = [&](int s) { return smem + C::kRing0 + s * C::kKSlotBytes; };
  auto vslot = [&](int s) { return smem + C::kVRing0 + s * C::kVSlotBytes; };
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (warp == kWarpProducer && lane == 0) {
    mbar_init(&bars[C::kBarQ], 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars[C::kBarK + s], 1);
      mbar_init(&bars[C::kBarKEmpty + s], 1);
      mbar_init(&bars[C::kBarV + s], 1);
      mbar_init(&bars[C::kBarVEmpty + s], 1);
    }
    for (int i = 0; i < kQT * 2; ++i) {
      mbar_init(&bars[C::kBarS + i], 1);
      mbar_init(&bars[C::kBarP + i], 128);
    }
    for (int t = 0; t < kQT; ++t) mbar_init(&bars[C::kBarO + t], 1);
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
      uint32_t need[kQT] = {0u, 0u};
      for (int t = 0; t < kQT; ++t) {
        for (int n = 0; n <= rt(t).n_last; ++n) need[t] |= kinds_of(t, n);
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
      int issued = 0;
      bool ok = true;
      for (int n = 0; n <= n_end; ++n) {
        const int s = n % C::kStages;
        const uint32_t j = n / C::kStages;
        // K tile n (every format some query tile routes it to)
        if (j > 0 &&
            !mbar_wait(&bars[C::kBarKEmpty + s], (j - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t kinds = kinds_of(0, n) | kinds_of(1, n);
        const int krow = start + n * kBN;
        uint8_t* ks = kslot(s);
        mbar_arrive_expect_tx(&bars[C::kBarK + s],
                              ((kinds & kKindF16) ? C::kK16Bytes : 0) +
                                  ((kinds & kKindI8) ? C::kK8Bytes : 0));
        if (kinds & kKindF16)
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(ks + c * kBN * 128, &p.tm_k, &bars[C::kBarK + s],
                        c * 64, krow, hk);
        if (kinds & kKindI8)
          tma_load_3d(ks + C::kK8Off, &p.tm_k8, &bars[C::kBarK + s], 0, krow,
                      hk);
        issued = n + 1;
        // V tile n
        if (j > 0 &&
            !mbar_wait(&bars[C::kBarVEmpty + s], (j - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&bars[C::kBarV + s], C::kVBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(vslot(s) + c * kBN * 128, &p.tm_v, &bars[C::kBarV + s],
                      c * 64, krow, hk);
      }
      if (!ok) {
        fail();
        // Let the copies already in flight land before the CTA exits.
        mbar_wait(&bars[C::kBarQ], 0, nullptr);
        // (a V copy is issued only after its K copy; waiting on both rings'
        // last fills covers every copy in flight, a V that was never issued
        // ends the wait by its time limit)
        for (int n = max(0, issued - C::kStages); n < issued; ++n) {
          const int s = n % C::kStages;
          mbar_wait(&bars[C::kBarK + s], (n / C::kStages) & 1, nullptr);
          mbar_wait(&bars[C::kBarV + s], (n / C::kStages) & 1, nullptr);
        }
      }
    }
  } else if (warp == kWarpMma) {
    // =================== MMA issuer (one thread) ===================
    if (lane == 0) {
      constexpr uint32_t idesc_qk16 = instr_desc(1, 0, 0, 0, 0, kBN, kBM);
      constexpr uint32_t idesc_qk8 = instr_desc(2, 1, 1, 0, 0, kBN, kBM);
      constexpr uint32_t idesc_pv = instr_desc(1, 0, 0, 0, 1, D, kBM);
      bool ok = mbar_wait(&bars[C::kBarQ], 0, abort_flag);
      tc_fence_after();

      // S_t(n) = Q_t K(n)^T on the path(s) tile t routes key tile n to.
      auto issue_qk = [&](int t, int n) -> bool {
        if (n > rt(t).n_last) return true;
        const uint32_t kinds = kinds_of(t, n);
        const int s = n % C::kStages;
        if (!mbar_wait(&bars[C::kBarK + s], (n / C::kStages) & 1, abort_flag))
          return false;
        tc_fence_after();
        const int slot = n % C::kSlots;
        const uint32_t kb = smem_u32(kslot(s));
        const uint32_t tbase = tmem + t * C::kTileCols;
        if (kinds & kKindF16) {
          const uint32_t q16 = smem_u32(sQ(t));
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_f16_ss(tbase + C::s16_col(slot), desc_k_f16(q16, kBM, ks),
                       desc_k_f16(kb, kBN, ks), idesc_qk16, ks > 0 ? 1u : 0u);
        }
        if (kinds & kKindI8) {
          const uint32_t q8 = smem_u32(sQ8(t));
#pragma unroll
          for (int ks = 0; ks < D / 32; ++ks)
            mma_i8_ss(tbase + C::s8_col(slot), desc_k_i8<D>(q8, ks),
                      desc_k_i8<D>(kb + C::kK8Off, ks), idesc_qk8,
                      ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars[C::kBarS + t * 2 + slot]);
        return true;
      };
      // O_t += P_t(n) V(n), P_t(n) read from the fp16 S columns in TMEM.
      auto issue_pv = [&](int t, int n) -> bool {
        if (n > rt(t).n_last) return true;
        const int s = n % C::kStages;
        const int slot = n % C::kSlots;
        if (!mbar_wait(&bars[C::kBarP + t * 2 + slot], (n / C::kSlots) & 1,
                       abort_flag))
          return false;
        if (!mbar_wait(&bars[C::kBarV + s], (n / C::kStages) & 1, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t vb = smem_u32(vslot(s));
        const uint32_t tbase = tmem + t * C::kTileCols;
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks)
          mma_f16_ts(tbase + C::kOCol, tbase + C::s16_col(slot) + ks * 8,
                     desc_v(vb, ks), idesc_pv, (n > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&bars[C::kBarO + t]);
        return true;
      };

      // Q K^T runs kSlots key tiles ahead of P V on each query tile.  A K
      // slot is released once both tiles' Q K^T of it completed, a V slot
      // once both tiles' P V did.
      for (int a = 0; a < C::kSlots && ok; ++a) {
        for (int t = 0; t < kQT && ok; ++t) ok = issue_qk(t, a);
        if (ok && a <= n_end) mma_commit(&bars[C::kBarKEmpty + a % C::kStages]);
      }
      for (int n = 0; n <= n_end && ok; ++n) {
        const int na = n + C::kSlots;
        for (int t = 0; t < kQT && ok; ++t) {
          ok = issue_pv(t, n);
          if (ok) ok = issue_qk(t, na);
        }
        if (ok) {
          mma_commit(&bars[C::kBarVEmpty + n % C::kStages]);
          if (na <= n_end) mma_commit(&bars[C::kBarKEmpty + na % C::kStages]);
        }
      }
      if (!ok) fail();
      // Drain: every MMA issued above has finished once this completes.
      mma_commit(&bars[C::kBarDrain]);
      mbar_wait(&bars[C::kBarDrain], 0, nullptr);
    }
    __syncwarp();
  } else {
    // ============ softmax warpgroups: warps 0-3 tile 0, 4-7 tile 1 ============
    const int t = warp >> 2;             // query tile of this warpgroup
    const int r = threadIdx.x & 127;     // score row = TMEM lane
    const TileRoute R = rt(t);
    if (R.n_last >= 0) {
      const int r_local = row_base + t * kBM + r;
      const bool valid = r_local < len;
      const int half = DUAL ? (r >> 6) : 0;
      const uint64_t my_w = half ? R.w1 : R.w0;
      const int my_nl = half ? R.nl1 : R.nl0;
      const uint32_t tbase = tmem + t * C::kTileCols;
      const uint32_t lane_addr =
          tbase + (static_cast<uint32_t>((warp & 3) * 32) << 16);
      const int key_lim = min(r_local, len - 1);  // keys j <= key_lim legal
      float sq = 0.0f;
      if (routed)
        sq = p.q_scale[(static_cast<size_t>(h) * p.batch + b) * p.nbq +
                       key_lim / p.quant_block_q];
      const float* kscale =
          routed ? p.k_scale + (static_cast<size_t>(hk) * p.batch + b) * p.nbk
                 : nullptr;
      // The K scale of tile n+1 is fetched while tile n is processed.
      float sk_next = routed ? kscale[0] : 0.0f;

      float m_run = -CUDART_INF_F;
      float l_run = 0.0f;
      bool ok = true;
      for (int n = 0; n <= R.n_last; ++n) {
        const int slot = n % C::kSlots;
        const float sk = sk_next;
        if (routed && n < R.n_last)
          sk_next = kscale[((n + 1) * kBN) / p.quant_block_k];
        // Exits stay warp-uniform: the tcgen05.ld/st below are .sync.aligned.
        const bool got_s = mbar_wait(&bars[C::kBarS + t * 2 + slot],
                                     (n / C::kSlots) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, got_s)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kinds = kinds_of(t, n);
        const bool mine_i8 = (n <= my_nl)
                                 ? (((my_w >> (n / tpb)) & 1ull) != 0)
                                 : ((kinds & kKindI8) != 0);
        const int col = mine_i8 ? C::s8_col(slot) : C::s16_col(slot);
        uint32_t sv[kBN];
        tmem_ld32(lane_addr + col, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(lane_addr + col + 32,
                  *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_ld_wait();

        if (p.qk_dump && mine_i8 && n <= my_nl && valid) {
          const int rrow = r_local / p.route_bm;
          const int rr = r_local - rrow * p.route_bm;
          const int key0 = n * kBN;
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
          for (int j = 0; j < kBN; ++j)
            if (j < keys_left) dst[j] = static_cast<int32_t>(sv[j]);
        }

        // Scores in log2 units are x_j = S_j * c with c > 0 (c = 0 only for
        // an all-zero quantisation block).
        float c = p.scale_log2;
        if (mine_i8) {
          c *= sq * sk;
          // INT32 accumulators to fp32, exactly (|acc| <= 127^2 d < 2^22),
          // on the integer and FMA pipes rather than the conversion unit.
#pragma unroll
          for (int j = 0; j < kBN; j += 2) {
            const float2 biased =
                make_float2(__uint_as_float(sv[j] + kIntBiasBits),
                            __uint_as_float(sv[j + 1] + kIntBiasBits));
            const float2 v =
                __fadd2_rn(biased, make_float2(-kIntBias, -kIntBias));
            sv[j] = __float_as_uint(v.x);
            sv[j + 1] = __float_as_uint(v.y);
          }
        }
        auto f = [&](int j) { return __uint_as_float(sv[j]); };
        const int lim = key_lim - n * kBN;  // columns j <= lim are legal
        const bool full = lim >= kBN - 1;
        if (!full) {
#pragma unroll
          for (int j = 0; j < kBN; ++j)
            if (j > lim) sv[j] = __float_as_uint(-CUDART_INF_F);
        }
        // Row max: four independent chains of 3-input max.
        float a0 = -CUDART_INF_F, a1 = -CUDART_INF_F, a2 = -CUDART_INF_F,
              a3 = -CUDART_INF_F;
#pragma unroll
        for (int j = 0; j < kBN; j += 8) {
          a0 = fmax3(a0, f(j), f(j + 1));
          a1 = fmax3(a1, f(j + 2), f(j + 3));
          a2 = fmax3(a2, f(j + 4), f(j + 5));
          a3 = fmax3(a3, f(j + 6), f(j + 7));
        }
        const float mx = fmax3(a0, a1, fmaxf(a2, a3));
        const float m_tile = (mx == -CUDART_INF_F) ? -CUDART_INF_F : mx * c;
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
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t o[32];
              tmem_ld32(lane_addr + C::kOCol + c0, o);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j)
                o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
              tmem_st32(lane_addr + C::kOCol + c0, o);
            }
          }
        }
        if (need) {
          l_run *= ex2_approx(m_run - m_new);
          m_run = m_new;
        }
        // P = 2^(x - m) as fp16 pairs in the first 32 columns of the fp16 S
        // slot (key 2i in the low half of column i); four packed partial sums.
        const float2 c2 = make_float2(c, c);
        const float2 nm2 = make_float2(-m_run, -m_run);
        float2 ps0 = make_float2(0.f, 0.f), ps1 = ps0, ps2 = ps0, ps3 = ps0;
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int j = 2 * i;
          const float2 x = __ffma2_rn(make_float2(f(j), f(j + 1)), c2, nm2);
          float2 pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          if (!full) {  // masked keys: exactly 0 (also when c == 0)
            pr.x = (j <= lim) ? pr.x : 0.0f;
            pr.y = (j + 1 <= lim) ? pr.y : 0.0f;
          }
          switch (i & 3) {
            case 0: ps0 = __fadd2_rn(ps0, pr); break;
            case 1: ps1 = __fadd2_rn(ps1, pr); break;
            case 2: ps2 = __fadd2_rn(ps2, pr); break;
            default: ps3 = __fadd2_rn(ps3, pr); break;
          }
          pk[i] = pack_half2(pr.x, pr.y);
        }
        tmem_st32(lane_addr + C::s16_col(slot), pk);
        const float2 s4 = __fadd2_rn(__fadd2_rn(ps0, ps1), __fadd2_rn(ps2, ps3));
        l_run += s4.x + s4.y;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars[C::kBarP + t * 2 + slot]);
      }

      const bool got_last =
          ok && mbar_wait(&bars[C::kBarO + t], R.n_last & 1, abort_flag);
      if (__all_sync(0xffffffffu, got_last)) {
        tc_fence_after();
        const float inv_l = 1.0f / l_run;
        uint16_t* orow =
            p.out + (static_cast<size_t>(start + r_local) * p.hq + h) * D;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(lane_addr + C::kOCol + c0, o);
          tmem_ld_wait();
          uint32_t hv[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            hv[j] = pack_half2(__uint_as_float(o[2 * j]) * inv_l,
                               __uint_as_float(o[2 * j + 1]) * inv_l);
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(hv[4 * v], hv[4 * v + 1], hv[4 * v + 2],
                                  hv[4 * v + 3]);
          }
        }
        if (p.lse && valid)
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
  const int pairs = (p.max_seqlen + kQT * kBM - 1) / (kQT * kBM);
  dim3 grid(p.hq, pairs, p.batch);
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
