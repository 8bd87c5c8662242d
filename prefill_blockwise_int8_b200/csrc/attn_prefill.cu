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
// B200 design (one CTA = one 128-row query tile of one head):
//   warp 4      TMA producer: Q / Q8 once, then per key tile the K tile in the
//               routed format (fp16 or int8) and the fp16 V tile, into a ring
//               of shared-memory stages;
//   warp 5      one thread issues tcgen05.mma: S = Q K^T (kind::f16 into f32
//               TMEM) or S = Q8 K8^T (kind::i8 into s32 TMEM), then
//               O += P V with P read from TMEM (kind::f16, f32 accumulator);
//   warps 0-3   softmax warpgroup, thread t owns score row t (TMEM lane t):
//               per-tile rescale of INT32 scores by q_scale * k_scale, causal
//               and end-of-sequence masking, running max / sum in fp32, lazy
//               rescale of O in TMEM when the max grows by more than 2^8,
//               P written back to TMEM as fp16, then the final O / l epilogue.
// S is double-buffered in TMEM so that Q K^T of tile n+1 runs on the tensor
// cores while the softmax warps work on tile n.
//
// With 64-row routing words (block_m = 64) a 128-row compute tile covers two
// routing rows; a key tile whose two halves route differently is computed
// on both paths into separate TMEM buffers and each row reads its own.
#include <cuda.h>
#include <cuda_fp16.h>
#include <math_constants.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace tilemix {
namespace {

constexpr int kBM = 128;          // compute-tile rows = TMEM lanes = MMA M
constexpr int kThreads = 192;     // 4 softmax warps + producer + MMA
constexpr int kSmemBudget = 232448;  // max dynamic smem per block on sm_100
constexpr uint32_t kKindF16 = 1, kKindI8 = 2;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when the
                                           // row max grows by more than 2^8

__host__ __device__ constexpr int align1k(int x) { return (x + 1023) & ~1023; }
__host__ __device__ constexpr int pow2_cols(int x) {
  return x <= 32 ? 32 : x <= 64 ? 64 : x <= 128 ? 128 : x <= 256 ? 256 : 512;
}

template <int D, int BN, bool DUAL>
struct Cfg {
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kQ8Bytes = kBM * D;
  static constexpr int kK16Bytes = BN * D * 2;
  static constexpr int kK8Bytes = BN * D;
  static constexpr int kVBytes = BN * D * 2;
  // Without two routing rows a tile needs one K format only, so the fp16
  // and int8 K tiles share one slot.
  static constexpr int kK8Off = DUAL ? align1k(kK16Bytes) : 0;
  static constexpr int kVOff = align1k(DUAL ? kK8Off + kK8Bytes : kK16Bytes);
  static constexpr int kStageBytes = align1k(kVOff + kVBytes);
  static constexpr int kQ8Off = align1k(kQBytes);
  static constexpr int kStage0 = align1k(kQ8Off + kQ8Bytes);
  static constexpr int kBarBytes = 256;
  static constexpr int kStagesFit =
      (kSmemBudget - 1024 - kBarBytes - kStage0) / kStageBytes;
  static constexpr int kStages = kStagesFit > 4 ? 4 : kStagesFit;
  static_assert(kStages >= 2, "shared memory too small for two stages");
  static constexpr int kBarOff = kStage0 + kStages * kStageBytes;
  static constexpr int kSmem = kBarOff + kBarBytes + 1024;  // + align slack
  // TMEM columns: S slots (f32 / s32, BN columns each), then O (D columns).
  static constexpr int kSlots = DUAL ? 4 : 2;
  static constexpr int kOCol = kSlots * BN;
  static constexpr int kTmemCols = pow2_cols(kOCol + D);
  static_assert(kOCol + D <= 512, "TMEM overflow");
  // barrier indices
  static constexpr int kBarQ = 0;
  static constexpr int kBarK = 1;
  static constexpr int kBarV = kBarK + kStages;
  static constexpr int kBarKVEmpty = kBarV + kStages;
  static constexpr int kBarS = kBarKVEmpty + kStages;  // 2
  static constexpr int kBarP = kBarS + 2;              // 2
  static constexpr int kBarO = kBarP + 2;              // 1
  static constexpr int kBarDrain = kBarO + 1;          // 1
  static constexpr int kNumBars = kBarDrain + 1;
  static_assert(kNumBars * 8 + 16 <= kBarBytes, "barrier area");
  static constexpr int s16_col(int slot) { return slot * BN; }
  static constexpr int s8_col(int slot) { return (DUAL ? 2 + slot : slot) * BN; }
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

// MN-major fp16 V tile (BN keys x D) stored as D/64 chunks [BN][128 B];
// ks = K-step of 16 keys.  LBO = chunk stride, SBO = 8 keys.
template <int BN>
__device__ __forceinline__ uint64_t desc_v(uint32_t base, int ks) {
  return smem_desc(base + ks * 16 * 128, BN * 128, 1024, kSwizzle128);
}

template <int D, int BN, bool DUAL>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  using C = Cfg<D, BN, DUAL>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.x;
  const int b = blockIdx.y;
  const int mc = gridDim.z - 1 - blockIdx.z;  // longest query tiles first

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
  const int row0 = mc * kBM;
  if (row0 >= len) return;
  const int hk = p.head_map ? p.head_map[h] : h / p.heads_per_kv;
  if (hk < 0 || hk >= p.hkv) {
    if (threadIdx.x == 0) report_status(p.status, kStatusBadSeqlens);
    return;
  }
  const int last_row = min(row0 + kBM - 1, len - 1);
  const int n_last = last_row / BN;  // last key tile with a legal key

  // Routing words.  With 64-row routing, half 0 = rows 0..63 of the tile.
  const size_t wbase = (static_cast<size_t>(b) * p.hkv + hk) * p.tm_route;
  uint64_t w0, w1 = 0;
  int nl0, nl1 = -1;
  const bool routed = !p.fp16_only;  // the mask may be NULL otherwise
  if (DUAL) {
    w0 = routed ? p.mask[wbase + 2 * mc] : 0;
    nl0 = min(row0 + 63, len - 1) / BN;
    if (row0 + 64 < len) {
      w1 = routed ? p.mask[wbase + 2 * mc + 1] : 0;
      nl1 = n_last;
    }
  } else {
    w0 = routed ? p.mask[wbase + mc] : 0;
    nl0 = n_last;
  }
  const int group = p.group;
  // Which score paths key tile n needs (bit 0: FP16, bit 1: INT8).
  auto tile_kinds = [&](int n) -> uint32_t {
    const int gi = n / group;
    uint32_t k = 0;
    if (n <= nl0) k |= ((w0 >> gi) & 1ull) ? kKindI8 : kKindF16;
    if (DUAL && n <= nl1) k |= ((w1 >> gi) & 1ull) ? kKindI8 : kKindF16;
    return k;
  };

  // ---- shared memory carve-up ----
  uint8_t* sQ = smem;
  uint8_t* sQ8 = smem + C::kQ8Off;
  auto stage_ptr = [&](int s) { return smem + C::kStage0 + s * C::kStageBytes; };
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (warp == 4 && lane == 0) {
    mbar_init(&bars[C::kBarQ], 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars[C::kBarK + s], 1);
      mbar_init(&bars[C::kBarV + s], 1);
      mbar_init(&bars[C::kBarKVEmpty + s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[C::kBarS + i], 1);
      mbar_init(&bars[C::kBarP + i], 128);
    }
    mbar_init(&bars[C::kBarO], 1);
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
  if (warp == 5) {
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

  if (warp == 4) {
    // =================== TMA producer ===================
    if (lane == 0) {
      uint32_t all = 0;
      for (int n = 0; n <= n_last; ++n) all |= tile_kinds(n);
      const int qrow = start + row0;
      mbar_arrive_expect_tx(&bars[C::kBarQ],
                            ((all & kKindF16) ? C::kQBytes : 0) +
                                ((all & kKindI8) ? C::kQ8Bytes : 0));
      if (all & kKindF16)
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sQ + c * kBM * 128, &p.tm_q, &bars[C::kBarQ], c * 64,
                      qrow, h);
      if (all & kKindI8) tma_load_3d(sQ8, &p.tm_q8, &bars[C::kBarQ], 0, qrow, h);
      int issued = 0;
      bool ok = true;
      for (int n = 0; n <= n_last && ok; ++n) {
        const int s = n % C::kStages;
        const int j = n / C::kStages;
        if (j > 0 && !mbar_wait(&bars[C::kBarKVEmpty + s], (j - 1) & 1,
                                abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t kinds = tile_kinds(n);
        const int krow = start + n * BN;
        uint8_t* st = stage_ptr(s);
        mbar_arrive_expect_tx(&bars[C::kBarK + s],
                              ((kinds & kKindF16) ? C::kK16Bytes : 0) +
                                  ((kinds & kKindI8) ? C::kK8Bytes : 0));
        if (kinds & kKindF16)
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(st + c * BN * 128, &p.tm_k, &bars[C::kBarK + s],
                        c * 64, krow, hk);
        if (kinds & kKindI8)
          tma_load_3d(st + C::kK8Off, &p.tm_k8, &bars[C::kBarK + s], 0, krow,
                      hk);
        mbar_arrive_expect_tx(&bars[C::kBarV + s], C::kVBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(st + C::kVOff + c * BN * 128, &p.tm_v,
                      &bars[C::kBarV + s], c * 64, krow, hk);
        issued = n + 1;
      }
      if (!ok) {
        fail();
        // Let the copies already in flight land before the CTA exits.
        mbar_wait(&bars[C::kBarQ], 0, nullptr);
        for (int n = max(0, issued - C::kStages); n < issued; ++n) {
          const int s = n % C::kStages;
          mbar_wait(&bars[C::kBarK + s], (n / C::kStages) & 1, nullptr);
          mbar_wait(&bars[C::kBarV + s], (n / C::kStages) & 1, nullptr);
        }
      }
    }
  } else if (warp == 5) {
    // =================== MMA issuer (one thread) ===================
    if (lane == 0) {
      constexpr uint32_t idesc_qk16 = instr_desc(1, 0, 0, 0, 0, BN, kBM);
      constexpr uint32_t idesc_qk8 = instr_desc(2, 1, 1, 0, 0, BN, kBM);
      constexpr uint32_t idesc_pv = instr_desc(1, 0, 0, 0, 1, D, kBM);
      const uint32_t q16 = smem_u32(sQ);
      const uint32_t q8 = smem_u32(sQ8);
      bool ok = mbar_wait(&bars[C::kBarQ], 0, abort_flag);
      tc_fence_after();

      auto issue_pv = [&](int t) -> bool {
        const int s = t % C::kStages;
        const int slot = t & 1;
        if (!mbar_wait(&bars[C::kBarP + slot], (t >> 1) & 1, abort_flag))
          return false;
        if (!mbar_wait(&bars[C::kBarV + s], (t / C::kStages) & 1, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t vb = smem_u32(stage_ptr(s) + C::kVOff);
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks)
          mma_f16_ts(tmem + C::kOCol, tmem + C::s16_col(slot) + ks * 8,
                     desc_v<BN>(vb, ks), idesc_pv, (t > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&bars[C::kBarO]);
        mma_commit(&bars[C::kBarKVEmpty + s]);
        return true;
      };

      for (int n = 0; n <= n_last && ok; ++n) {
        const int s = n % C::kStages;
        const int slot = n & 1;
        if (!mbar_wait(&bars[C::kBarK + s], (n / C::kStages) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kinds = tile_kinds(n);
        const uint32_t kb = smem_u32(stage_ptr(s));
        if (kinds & kKindF16) {
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_f16_ss(tmem + C::s16_col(slot), desc_k_f16(q16, kBM, ks),
                       desc_k_f16(kb, BN, ks), idesc_qk16, ks > 0 ? 1u : 0u);
        }
        if (kinds & kKindI8) {
#pragma unroll
          for (int ks = 0; ks < D / 32; ++ks)
            mma_i8_ss(tmem + C::s8_col(slot), desc_k_i8<D>(q8, ks),
                      desc_k_i8<D>(kb + C::kK8Off, ks), idesc_qk8,
                      ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars[C::kBarS + slot]);
        if (n > 0 && !issue_pv(n - 1)) ok = false;
      }
      if (ok) ok = issue_pv(n_last);
      if (!ok) fail();
      // Drain: every MMA issued above has finished once this completes.
      mma_commit(&bars[C::kBarDrain]);
      mbar_wait(&bars[C::kBarDrain], 0, nullptr);
    }
    __syncwarp();
  } else {
    // =================== softmax warpgroup (warps 0-3) ===================
    const int t = threadIdx.x;  // score row inside the tile = TMEM lane
    const int r_local = row0 + t;
    const bool valid = r_local < len;
    const int half = DUAL ? (t >> 6) : 0;
    const uint64_t my_w = half ? w1 : w0;
    const int my_nl = half ? nl1 : nl0;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int r_clamped = min(r_local, len - 1);
    float sq = 0.0f;
    if (!p.fp16_only)
      sq = p.q_scale[(static_cast<size_t>(h) * p.batch + b) * p.nbq +
                     r_clamped / p.quant_block_q];
    const float* kscale =
        p.fp16_only ? nullptr
                    : p.k_scale + (static_cast<size_t>(hk) * p.batch + b) * p.nbk;
    const int key_lim = r_clamped;  // keys j <= key_lim are legal for this row

    float m_run = -CUDART_INF_F;
    float l_run = 0.0f;
    bool ok = true;
    for (int n = 0; n <= n_last; ++n) {
      const int slot = n & 1;
      // Exits stay warp-uniform: the tcgen05.ld/st below are .sync.aligned.
      const bool got_s = mbar_wait(&bars[C::kBarS + slot], (n >> 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, got_s)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t kinds = tile_kinds(n);
      const bool mine_i8 = (n <= my_nl) ? (((my_w >> (n / group)) & 1ull) != 0)
                                        : ((kinds & kKindI8) != 0);
      const int col = mine_i8 ? C::s8_col(slot) : C::s16_col(slot);
      uint32_t sv[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c)
        tmem_ld32(lane_addr + col + c * 32,
                  *reinterpret_cast<uint32_t(*)[32]>(&sv[c * 32]));
      tmem_ld_wait();

      if (p.qk_dump && mine_i8 && n <= my_nl && valid) {
        const int rrow = r_local / p.route_bm;
        const int rr = r_local - rrow * p.route_bm;
        int32_t* dst =
            p.qk_dump +
            ((((static_cast<size_t>(b) * p.hq + h) * p.tm_route + rrow) *
                  p.tn_max +
              n) *
                 p.route_bm +
             rr) *
                BN;
        const int keys_left = len - n * BN;  // keys inside the sequence
        for (int j = 0; j < BN; ++j)
          if (j < keys_left) dst[j] = static_cast<int32_t>(sv[j]);
      }

      // Scores in log2 units are x_j = S_j * c with c > 0 (or 0 for an
      // all-zero quantisation block).
      float c = p.scale_log2;
      if (mine_i8) c *= sq * kscale[(n * BN) / p.quant_block_k];
      // Scores as fp32, kept as raw bits in sv (INT32 accumulators convert
      // exactly: |acc| <= 127^2 * d < 2^24).
      if (mine_i8) {
#pragma unroll
        for (int j = 0; j < BN; ++j)
          sv[j] = __float_as_uint(static_cast<float>(static_cast<int32_t>(sv[j])));
      }
      auto f = [&](int j) { return __uint_as_float(sv[j]); };
      const int lim = key_lim - n * BN;  // columns j <= lim are legal
      float m_tile;
      if (lim >= BN - 1) {
        float mx = f(0);
#pragma unroll
        for (int j = 1; j < BN; ++j) mx = fmaxf(mx, f(j));
        m_tile = mx * c;
      } else {
        m_tile = -CUDART_INF_F;
#pragma unroll
        for (int j = 0; j < BN; ++j)
          if (j <= lim) m_tile = fmaxf(m_tile, f(j) * c);
      }
      const float m_new = fmaxf(m_run, m_tile);
      const bool need = m_new > m_run + kRescaleThreshold;

      if (n > 0) {
        // O holds P V of every tile before n once PV(n-1) completed.
        const bool got_o = mbar_wait(&bars[C::kBarO], (n - 1) & 1, abort_flag);
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
      // P = 2^(x - m) as fp16 pairs over the first BN/2 columns of the S
      // slot (key 2i in the low half of column i), 64 keys at a time.
      float psum = 0.0f;
#pragma unroll
      for (int j0 = 0; j0 < BN; j0 += 64) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int j = j0 + 2 * i;
          const float p0 =
              (j <= lim) ? ex2_approx(fmaf(f(j), c, -m_run)) : 0.0f;
          const float p1 =
              (j + 1 <= lim) ? ex2_approx(fmaf(f(j + 1), c, -m_run)) : 0.0f;
          psum += p0 + p1;
          pk[i] = pack_half2(p0, p1);
        }
        tmem_st32(lane_addr + C::s16_col(slot) + j0 / 2, pk);
      }
      l_run += psum;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars[C::kBarP + slot]);
    }

    const bool got_last =
        ok && mbar_wait(&bars[C::kBarO], n_last & 1, abort_flag);
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

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, C::kTmemCols);
}

template <int D, int BN, bool DUAL>
cudaError_t launch_one(const AttnParams& p, cudaStream_t stream) {
  using C = Cfg<D, BN, DUAL>;
  auto kern = attn_fwd_kernel<D, BN, DUAL>;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const int tmc = (p.max_seqlen + kBM - 1) / kBM;
  dim3 grid(p.hq, p.batch, tmc);
  kern<<<grid, kThreads, C::kSmem, stream>>>(p);
  return cudaGetLastError();
}

template <int D, int BN, bool DUAL>
int smem_of() {
  return Cfg<D, BN, DUAL>::kSmem;
}

}  // namespace

cudaError_t launch_attn_prefill(const AttnParams& p, const AttnLaunchShape& s,
                                cudaStream_t stream) {
  if (s.head_dim == 128) {
    if (s.block_n == 128 && !s.dual) return launch_one<128, 128, false>(p, stream);
    if (s.block_n == 64 && !s.dual) return launch_one<128, 64, false>(p, stream);
    if (s.block_n == 64 && s.dual) return launch_one<128, 64, true>(p, stream);
  } else if (s.head_dim == 64) {
    if (s.block_n == 128 && !s.dual) return launch_one<64, 128, false>(p, stream);
    if (s.block_n == 64 && !s.dual) return launch_one<64, 64, false>(p, stream);
    if (s.block_n == 64 && s.dual) return launch_one<64, 64, true>(p, stream);
  }
  return cudaErrorInvalidValue;
}

int attn_smem_bytes(const AttnLaunchShape& s) {
  if (s.head_dim == 128) {
    if (s.block_n == 128 && !s.dual) return smem_of<128, 128, false>();
    if (s.block_n == 64 && !s.dual) return smem_of<128, 64, false>();
    if (s.block_n == 64 && s.dual) return smem_of<128, 64, true>();
  } else if (s.head_dim == 64) {
    if (s.block_n == 128 && !s.dual) return smem_of<64, 128, false>();
    if (s.block_n == 64 && !s.dual) return smem_of<64, 64, false>();
    if (s.block_n == 64 && s.dual) return smem_of<64, 64, true>();
  }
  return -1;
}

}  // namespace tilemix
