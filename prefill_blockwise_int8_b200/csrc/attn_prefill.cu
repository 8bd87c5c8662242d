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
//   warp 16     TMA producer: Q and/or Q8 of its query tiles once, then per
//               key tile the K tile in every format a query tile routes some
//               of it to (fp16 and/or int8) and the fp16 V tile;
//   warp 17     one thread issues tcgen05.mma: S_t = Q_t K^T (kind::f16, f32
//               in TMEM) or Q8_t K8^T (kind::i8, s32 in TMEM) per 64-key half
//               of the tile (one N = 128 instruction chain when both halves
//               take the same path), and O_t += P_t V with P_t read from TMEM
//               (kind::f16, f32 TMEM accumulator);
//   warps 0-15  softmax: warpgroups 2t and 2t+1 serve query tile t, one
//               thread per score row (= TMEM lane), keys 0..63 and 64..127
//               of each row, combining row max and sum through shared
//               memory; both tiles' warpgroups run at once, so every SM
//               sub-partition holds four softmax warps.  Per tile: INT32
//               scores rescaled by q_scale * k_scale, causal /
//               end-of-sequence masking, running max and sum in fp32, lazy
//               rescale of O in TMEM when the max grows by more than 2^8,
//               P back to TMEM as fp16; then O / l.
// 128-key tiles keep every FP16 MMA at N = 128: on sm_100a a kind::f16
// M128 K16 instruction costs about the same at N = 64 as at N = 128.
#include <cuda.h>
#include <cuda_fp16.h>
#include <climits>
#include <math_constants.h>
#include <stdint.h>

#include "attn_common.cuh"
#include "internal.h"
#include "ptx.cuh"
#include "quant_code.cuh"

namespace tilemix {
namespace {

constexpr int kBM = 128;     // query rows per tile = TMEM lanes = MMA M
constexpr int kBN = 128;     // keys per compute tile
constexpr int kHalf = 64;    // routing granularity inside a compute tile
constexpr int kWarpProducer = 16;
constexpr int kWarpMma = 17;
constexpr int kWarpConv = 18;  // two converter warps (modes 1 and 2)
// Operand modes: Q8/K8 and scales given (quantised once before the call),
// the INT8 KV cache (K8/V8 given, fp16 copies made on chip), or Q8/K8 and
// their scales made on chip from Q/K for INT8-routed tiles only.
constexpr int kModeGiven = 0, kModeKV8 = 1, kModeOnChip = 2;
// 16 softmax warps, producer, MMA issuer (+ two converter warps)
__host__ __device__ constexpr int threads_of(int mode) {
  return mode != kModeGiven ? 640 : 576;
}
constexpr int kSmemBudget = 232448;  // max dynamic smem per block on sm_100

__host__ __device__ constexpr int align1k(int x) { return (x + 1023) & ~1023; }

template <int D, bool DUAL, int MODE>
struct Cfg {
  static constexpr bool KV8 = MODE == kModeKV8;
  static constexpr bool QF = MODE == kModeOnChip;
  // DUAL (64-row routing words): a 128-row query tile may need both paths
  // for the same keys, so S has an fp16 and an int8 region and the CTA
  // holds one query tile.
  static constexpr int kQT = DUAL ? 1 : 2;
  static constexpr int kQBytes = kBM * D * 2;   // per query tile
  static constexpr int kQ8Bytes = kBM * D;
  static constexpr int kK16Bytes = kBN * D * 2;
  static constexpr int kK8Bytes = kBN * D;
  static constexpr int kVBytes = kBN * D * 2;
  // INT8 V tile, staged in the upper half of its V slot and converted in
  // place (row r of V8 lies exactly where chunk D/64 - 1 of row r of V goes
  // for d = 128; rows are converted by the thread that read them)
  static constexpr int kV8Bytes = kBN * D;
  static constexpr int kV8Off = D == 128 ? kVBytes - kV8Bytes : kVBytes;
  static constexpr int kQ8Off = kQT * kQBytes;
  static constexpr int kRing0 = align1k(kQ8Off + kQT * kQ8Bytes);
  static constexpr int kK8Off = align1k(kK16Bytes);
  // On-chip quantisation keeps its K8 tiles in a ring of their own, which
  // the converter warps fill from K in global memory ahead of the MMAs; its
  // K slots then hold fp16 K only.
  static constexpr int kKSlotBytes =
      QF ? align1k(kK16Bytes) : align1k(kK8Off + kK8Bytes);
  static constexpr int kK8Ring = QF ? 2 : 0;
  // (d = 64 stages V8 past the fp16 tile: there rows would overlap)
  static constexpr int kVSlotBytes =
      align1k(KV8 && D != 128 ? kVBytes + kBN * D : kVBytes);
  static constexpr int kRedBytes = 4096;  // max / sum exchange [tile][2][2][128]
  static constexpr int kBarBytes = 512;
  static constexpr int kAvail =
      kSmemBudget - 1024 - kBarBytes - kRedBytes - 128 - kRing0;
  // Two V slots (P V of every query tile must finish before a V slot
  // frees; one beside the on-chip K8 ring, whose V load has a whole softmax
  // pass to land), then as many K slots as fit (at most 3).
  static constexpr int kVStages = QF ? 1 : 2;
  static constexpr int kKFit =
      (kAvail - kVStages * kVSlotBytes - kK8Ring * kK8Bytes) / kKSlotBytes;
  static constexpr int kKStages = kKFit > 3 ? 3 : kKFit;
  static_assert(kKStages >= 1, "shared memory too small");
  static constexpr int kK8Ring0 = kRing0 + kKStages * kKSlotBytes;
  static constexpr int kVRing0 = kK8Ring0 + kK8Ring * kK8Bytes;
  static constexpr int kRedOff = kVRing0 + kVStages * kVSlotBytes;
  // on-chip quantisation: Q scales [2], K-scale ring [8], converter max
  // exchange [2][2]
  static constexpr int kAuxOff = kRedOff + kRedBytes;
  static constexpr int kAuxBytes = 128;
  // Q K^T halves of each query tile for the key tile in K slot s (written
  // by the producer before the slot's loads, read by the MMA issuer)
  static constexpr int kCodeOff = kAuxOff + 64;
  static constexpr int kSkRing = 8;
  static constexpr int kBarOff = kAuxOff + kAuxBytes;
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
  // P of warpgroup wg's 64 keys (32 columns): over the S columns it read
  // with two query tiles; in the spare columns with one.
  static constexpr int p_col(int wg) { return DUAL ? kP + 32 * wg : kHalf * wg; }
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
  static constexpr int kBarRed = kBarO + 2;            // [tile][parity]
  // INT8 KV cache: K slot holds its fp16 copy, V slot its fp16 V
  static constexpr int kBarOStage = kBarRed + 4;       // [tile]
  static constexpr int kBarKConv = kBarOStage + 2;     // [K slot]
  static constexpr int kBarVConv = kBarKConv + kKStages;  // [V slot]
  // on-chip quantisation: Q8 of a tile made, K scale of a key tile made,
  // converter-warp max exchange
  static constexpr int kBarQConv = kBarVConv + kVStages;  // [tile]
  static constexpr int kBarSK = kBarQConv + 2;            // [ring slot]
  static constexpr int kBarCvX = kBarSK + kSkRing;
  static constexpr int kBarK8Full = kBarCvX + 1;       // [K8 ring slot]
  static constexpr int kBarK8Empty = kBarK8Full + 2;   // [K8 ring slot]
  static constexpr int kBarDrain = kBarK8Empty + 2;
  static constexpr int kNumBars = kBarDrain + 1;
  static_assert(kNumBars * 8 + 16 <= kBarBytes, "barrier area");
};

// Row max of 64 scores held as raw bits (INT32 accumulators when I8, fp32
// otherwise).  With MASKED, columns j > hl are left out.  The masked /
// unmasked choice is made once per 64-key half, not per element.
template <bool I8, bool MASKED>
__device__ __forceinline__ float max64(const uint32_t (&sv)[64], int hl) {
  // eight independent 3-input chains of depth four, then a short tree
  if (I8) {
    auto g = [&](int j) {
      return (!MASKED || j <= hl) ? static_cast<int>(sv[j]) : INT_MIN;
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
    if (MASKED && hl < 0) return -CUDART_INF_F;
    return static_cast<float>(m);
  } else {
    auto g = [&](int j) {
      return (!MASKED || j <= hl) ? __uint_as_float(sv[j]) : -CUDART_INF_F;
    };
    float a[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = fmaxf(g(2 * k), g(2 * k + 1));
#pragma unroll
    for (int j = 16; j < 64; j += 16)
#pragma unroll
      for (int k = 0; k < 8; ++k)
        a[k] = fmax3(a[k], g(j + 2 * k), g(j + 2 * k + 1));
    return fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]),
                 fmaxf(a[6], a[7]));
  }
}

// P = 2^(S c - m) of 32 scores as 16 packed fp16 pairs (key 2i in the low
// half of pk[i]), added to four packed partial sums.  INT32 accumulators
// convert to fp32 exactly (|acc| <= 127^2 d < 2^22) by the bias trick, on
// the integer and FMA pipes rather than the conversion unit.  With MASKED,
// columns j > hl give exactly 0.  With TRACK, xmax accumulates the largest
// exponent S c - m over the legal columns.
template <bool I8, bool MASKED, bool TRACK>
__device__ __forceinline__ void exp32(const uint32_t (&sv)[32], float c,
                                      float m, int hl, uint32_t* pk,
                                      float2& ps0, float2& ps1, float2& ps2,
                                      float2& ps3, float& xmax) {
  const float2 c2 = make_float2(c, c);
  const float2 nm2 = make_float2(-m, -m);
  float xa = -CUDART_INF_F, xb = -CUDART_INF_F;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int j = 2 * i;
    float2 sc = make_float2(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1]));
    if (I8) {
      sc = __fadd2_rn(make_float2(__uint_as_float(sv[j] + kIntBiasBits),
                                  __uint_as_float(sv[j + 1] + kIntBiasBits)),
                      make_float2(-kIntBias, -kIntBias));
    }
    float2 x = __ffma2_rn(sc, c2, nm2);
    if (MASKED) {  // 2^-inf = 0, also when c == 0
      x.x = (j <= hl) ? x.x : -CUDART_INF_F;
      x.y = (j + 1 <= hl) ? x.y : -CUDART_INF_F;
    }
    if (TRACK) {
      if (i & 1) xb = fmax3(xb, x.x, x.y);
      else xa = fmax3(xa, x.x, x.y);
    }
    // P enters P V rounded to fp16; the row sum adds the same rounded
    // values, so O / l is a weighted mean with exactly the weights P V used
    const __half2 ph = __floats2half2_rn(ex2_approx(x.x), ex2_approx(x.y));
    const float2 pr = __half22float2(ph);
    switch (i & 3) {
      case 0: ps0 = __fadd2_rn(ps0, pr); break;
      case 1: ps1 = __fadd2_rn(ps1, pr); break;
      case 2: ps2 = __fadd2_rn(ps2, pr); break;
      default: ps3 = __fadd2_rn(ps3, pr); break;
    }
    pk[i] = *reinterpret_cast<const uint32_t*>(&ph);
  }
  if (TRACK) xmax = fmax3(xmax, xa, xb);
}

// Largest |x| of row rr of an fp16 tile stored as D/64 chunks of
// [128 rows][128 B] with the 128-byte swizzle.
template <int D>
__device__ __forceinline__ float row_absmax_f16(const uint8_t* tile, int rr) {
  __half2 m = __float2half2_rn(0.0f);
#pragma unroll
  for (int u = 0; u < D / 8; ++u) {
    const uint32_t o = (u / 8) * 128 * 128 + rr * 128 + (u % 8) * 16;
    const uint4 v = *reinterpret_cast<const uint4*>(tile + swz(o, 7));
    const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) m = __hmax2(m, __habs2(h[e]));
  }
  return fmaxf(__low2float(m), __high2float(m));
}

// 16 fp16 values (two 16-byte words) -> their 16 codes as one 16-byte word
// (code of value i in byte i), with the quantiser's exact definition.
__device__ __forceinline__ uint4 codes16(uint4 a, uint4 b, float s, float r) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t out[4];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    float f[8];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      half2_bits_to_float2(w[4 * hh + e], f[2 * e], f[2 * e + 1]);
    uint32_t cb[8];
    quant_codes8(f, s, r, cb);
    out[2 * hh] = pack_low_bytes4(cb[0], cb[1], cb[2], cb[3]);
    out[2 * hh + 1] = pack_low_bytes4(cb[4], cb[5], cb[6], cb[7]);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

// Codes of row rr of that fp16 tile into an INT8 tile of D-byte rows with
// the swizzle of mask sm (the layout the INT8 MMA reads), scale s, 1/s = r
// (a zero block has s = r = 0: codes 0).
template <int D>
__device__ __forceinline__ void quant_row(const uint8_t* tile16,
                                          uint8_t* tile8, uint32_t sm, int rr,
                                          float s, float r) {
#pragma unroll
  for (int v = 0; v < D / 16; ++v) {
    uint4 x[2];
#pragma unroll
    for (int hu = 0; hu < 2; ++hu) {
      const int u = 2 * v + hu;
      const uint32_t o = (u / 8) * 128 * 128 + rr * 128 + (u % 8) * 16;
      x[hu] = *reinterpret_cast<const uint4*>(tile16 + swz(o, 7));
    }
    *reinterpret_cast<uint4*>(tile8 + swz(rr * D + v * 16, sm)) =
        codes16(x[0], x[1], s, r);
  }
}

// Largest |x| of one contiguous fp16 row of D values in global memory.
template <int D>
__device__ __forceinline__ float row_absmax_global(const __half* row) {
  __half2 m = __float2half2_rn(0.0f);
#pragma unroll
  for (int u = 0; u < D / 8; ++u) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(row) + u);
    const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) m = __hmax2(m, __habs2(h[e]));
  }
  return fmaxf(__low2float(m), __high2float(m));
}

// Codes of one contiguous fp16 row in global memory (nullptr: a row past
// the sequence, codes 0) into row rr of an INT8 tile laid out as above.
template <int D>
__device__ __forceinline__ void quant_row_global(const __half* row,
                                                 uint8_t* tile8, uint32_t sm,
                                                 int rr, float s, float r) {
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int v = 0; v < D / 16; ++v) {
    const uint4 a = row ? __ldg(reinterpret_cast<const uint4*>(row) + 2 * v) : zero;
    const uint4 b = row ? __ldg(reinterpret_cast<const uint4*>(row) + 2 * v + 1) : zero;
    *reinterpret_cast<uint4*>(tile8 + swz(rr * D + v * 16, sm)) =
        codes16(a, b, s, r);
  }
}

// Routing state of one 128-row query tile.
struct TileRoute {
  uint64_t w0, w1;  // words of rows 0..63 / 64..127 (equal unless DUAL)
  int nl0, nl1;     // last legal 64-key block of each row half (-1: none)
  int n_last;       // last legal 128-key tile (-1: no rows)
};

template <int D, bool DUAL, int MODE>
__global__ void __launch_bounds__(threads_of(MODE), 1)
    attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  using C = Cfg<D, DUAL, MODE>;
  constexpr bool KV8 = MODE == kModeKV8;
  constexpr bool QF = MODE == kModeOnChip;
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
  auto rt = [&](int t) -> TileRoute { return t ? rt1 : rt0; };
  const int n_end = max(rt0.n_last, rt1.n_last);
  const int tpb = p.tiles_per_bit;  // 64-key blocks per routing bit
  // Paths query tile t needs for 64-key half kh of key tile n (0: none).
  auto kinds_of = [&](int t, int n, int kh) -> uint32_t {
    const TileRoute r = rt(t);
    const int n64 = 2 * n + kh;
    const int gi = n64 / tpb;
    uint32_t k = 0;
    if (n64 <= r.nl0) k |= ((r.w0 >> gi) & 1ull) ? kKindI8 : kKindF16;
    if (n64 <= r.nl1) k |= ((r.w1 >> gi) & 1ull) ? kKindI8 : kKindF16;
    return k;
  };
  // Q K^T of query tile t, key tile n: bits 0-1 the 64-key halves computed
  // on the FP16 path, bits 2-3 those on the INT8 path (0: no rows there).
  auto qk_code = [&](int t, int n) -> uint32_t {
    if (t >= kQT || n > rt(t).n_last) return 0u;
    const uint32_t k0 = kinds_of(t, n, 0);
    uint32_t k1 = kinds_of(t, n, 1);
    if (k1 == 0) k1 = k0;  // keys past every row: any path will do
    return ((k0 & kKindF16) ? 1u : 0u) | ((k1 & kKindF16) ? 2u : 0u) |
           ((k0 & kKindI8) ? 4u : 0u) | ((k1 & kKindI8) ? 8u : 0u);
  };
  uint32_t* qk_codes = reinterpret_cast<uint32_t*>(smem + C::kCodeOff);

  // ---- shared memory carve-up ----
  auto sQ = [&](int t) { return smem + t * C::kQBytes; };
  auto sQ8 = [&](int t) { return smem + C::kQ8Off + t * C::kQ8Bytes; };
  auto kslot = [&](int s) { return smem + C::kRing0 + s * C::kKSlotBytes; };
  auto vslot = [&](int s) { return smem + C::kVRing0 + s * C::kVSlotBytes; };
  // row max / sum exchange between the softmax warpgroups: [slot][wg][row]
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
      mbar_init(&bars[C::kBarP + i], 8);   // one arrival per softmax warp
      mbar_init(&bars[C::kBarO + i], 1);
      mbar_init(&bars[C::kBarOStage + i], 8);  // O of tile i staged
      mbar_init(&bars[C::kBarRed + 2 * i], 8);
      mbar_init(&bars[C::kBarRed + 2 * i + 1], 8);
    }
    if (KV8 || QF) {
      for (int s = 0; s < C::kKStages; ++s)
        mbar_init(&bars[C::kBarKConv + s], 2);  // the two converter warps
      for (int s = 0; s < C::kVStages; ++s)
        mbar_init(&bars[C::kBarVConv + s], 2);
      for (int i = 0; i < 2; ++i) mbar_init(&bars[C::kBarQConv + i], 2);
      for (int i = 0; i < C::kSkRing; ++i) mbar_init(&bars[C::kBarSK + i], 2);
      mbar_init(&bars[C::kBarCvX], 2);
      for (int i = 0; i < 2; ++i) {
        mbar_init(&bars[C::kBarK8Full + i], 2);   // the two converter warps
        mbar_init(&bars[C::kBarK8Empty + i], 1);  // MMA commit
      }
    }
    mbar_init(&bars[C::kBarDrain], 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_o);
    if (KV8) {
      tma_prefetch_desc(&p.tm_k8);
      tma_prefetch_desc(&p.tm_v8);
    } else {
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
    }
    if (routed && !QF) {  // the INT8 maps are empty in FP16-only mode
      tma_prefetch_desc(&p.tm_q8);
      if (!KV8) tma_prefetch_desc(&p.tm_k8);
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
      // Paths a query tile uses anywhere: its words' bits over the legal
      // groups (bit set: INT8 somewhere; bit clear: FP16 somewhere).
      auto need_of = [&](const TileRoute& r) -> uint32_t {
        auto legal = [&](int nl) -> uint64_t {
          if (nl < 0) return 0ull;
          const int gl = nl / tpb;  // last legal group
          return gl >= 63 ? ~0ull : ((1ull << (gl + 1)) - 1ull);
        };
        const uint64_t l0 = legal(r.nl0), l1 = legal(r.nl1);
        uint32_t k = 0;
        if ((r.w0 & l0) | (r.w1 & l1)) k |= kKindI8;
        if ((~r.w0 & l0) | (~r.w1 & l1)) k |= kKindF16;
        return k;
      };
      uint32_t qbytes = 0;
      uint32_t need[2] = {need_of(rt0), need_of(rt1)};
      // On-chip quantisation makes Q8 from Q: fetch Q for every tile.
      if (QF)
        for (int t = 0; t < 2; ++t) need[t] = need[t] ? kKindF16 : 0u;
      for (int t = 0; t < kQT; ++t)
        qbytes += ((need[t] & kKindF16) ? C::kQBytes : 0) +
                  ((need[t] & kKindI8) ? C::kQ8Bytes : 0);
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
      bool v_withheld = false;
      bool ok = true;
      for (int n = 0; n <= n_end && ok; ++n) {
        const int krow = start + n * kBN;
        // K tile n in every format some query tile routes part of it to
        const int ks = n % C::kKStages;
        const int jk = n / C::kKStages;
        // routing of this key tile, worked out before waiting for its slot
        const uint32_t code = qk_code(0, n) | (qk_code(1, n) << 4);
        uint32_t kinds = ((code & 0x33u) ? kKindF16 : 0u) |
                         ((code & 0xccu) ? kKindI8 : 0u);
        if (jk > 0 &&
            !mbar_wait(&bars[C::kBarKEmpty + ks], (jk - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        qk_codes[ks] = code;
        // The INT8 cache only holds K8 (the converters make the fp16 copy);
        // on-chip quantisation makes K8 from K.
        if (KV8) kinds = kKindI8;
        if (QF) kinds &= kKindF16;  // K8 comes from the converters' ring
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
        // Timeout-path test: V tile 0 is never loaded, so its barrier never
        // completes and the MMA issuer's bounded wait on it expires.
        if (n == 0 && p.test_expire_wait) {
          v_withheld = true;
          continue;
        }
        if (KV8) {
          mbar_arrive_expect_tx(&bars[C::kBarV + vs], C::kV8Bytes);
          tma_load_3d(vslot(vs) + C::kV8Off, &p.tm_v8, &bars[C::kBarV + vs], 0,
                      krow, hk);
        } else {
          mbar_arrive_expect_tx(&bars[C::kBarV + vs], C::kVBytes);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(vslot(vs) + c * kBN * 128, &p.tm_v,
                        &bars[C::kBarV + vs], c * 64, krow, hk);
        }
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
          if (!(n == 0 && v_withheld))
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
      // O in fp32, or (study flag) in fp16: one value in the low half of
      // each TMEM column either way
      const uint32_t idesc_pv = instr_desc(p.pv_f16_acc ? 0 : 1, 0, 0, 0, 1, D, kBM);
      bool ok = mbar_wait(&bars[C::kBarQ], 0, abort_flag);
      tc_fence_after();

      bool q8_ready0 = false, q8_ready1 = false;  // on-chip Q8 seen
      // Everything the issue path needs is worked out here, so the thread
      // (which shares its sub-partition with four softmax warps) spends as
      // few instructions as possible between a barrier and its MMAs:
      // descriptors are bases plus constant K-step offsets, the routing of
      // each key tile comes from the producer's code word.
      const int nl0 = rt0.n_last, nl1 = rt1.n_last;
      const uint64_t dq16_0 = desc_k_f16(smem_u32(sQ(0)), kBM * 128, 0);
      const uint64_t dq16_1 = desc_k_f16(smem_u32(sQ(kQT - 1)), kBM * 128, 0);
      const uint64_t dq8_0 = desc_k_i8<D>(smem_u32(sQ8(0)), 0);
      const uint64_t dq8_1 = desc_k_i8<D>(smem_u32(sQ8(kQT - 1)), 0);
      const uint64_t dk16_0 = desc_k_f16(smem_u32(kslot(0)), kBN * 128, 0);
      const uint64_t dk8_0 =
          desc_k_i8<D>(smem_u32(QF ? smem + C::kK8Ring0 : kslot(0) + C::kK8Off), 0);
      const uint64_t dv_0 = desc_v(smem_u32(vslot(0)), kBN * 128, 0);
      constexpr uint64_t kKSlotStep = C::kKSlotBytes >> 4;  // descriptor units
      constexpr uint64_t kVSlotStep = C::kVSlotBytes >> 4;
      // S_t(n) = Q_t K(n)^T, each 64-key half on the path(s) it routes to.
      auto issue_qk = [&](int t, int n) -> bool {
        if (n > (t ? nl1 : nl0)) return true;
        const int s = n % C::kKStages;
        if (!mbar_wait(&bars[C::kBarK + s], (n / C::kKStages) & 1, abort_flag))
          return false;
        tc_fence_after();
        // With converter warps, every key tile waits for them (the fp16 copy
        // of an INT8-cache K tile, or the on-chip K8): the K slot may only
        // free after they passed it, so they never miss a phase of its
        // full barrier.
        if (KV8 &&
            !mbar_wait(&bars[C::kBarKConv + s], (n / C::kKStages) & 1,
                       abort_flag))
          return false;
        const uint32_t code = (qk_codes[s] >> (4 * t)) & 0xfu;
        const uint32_t halves16 = code & 3u, halves8 = code >> 2;
        // On-chip quantisation: the converters' Q8 of this tile (once) and
        // the K8 of this key tile in ring slot n % 2.
        if (QF && halves8) {
          bool& qdone = t ? q8_ready1 : q8_ready0;
          if (!qdone && !mbar_wait(&bars[C::kBarQConv + t], 0, abort_flag))
            return false;
          qdone = true;
          if (!mbar_wait(&bars[C::kBarK8Full + (n & 1)], (n >> 1) & 1,
                         abort_flag))
            return false;
        }
        if (KV8 || QF) tc_fence_after();
        const uint32_t tb = tmem + t * C::kTileCols;
        const uint64_t slot_off = static_cast<uint64_t>(s) * kKSlotStep;
        if (halves16) {
          const uint64_t dq = t ? dq16_1 : dq16_0;
          // one N = 128 chain, or the single 64-key half that needs it
          const uint32_t hoff = (halves16 == 2u) ? 1u : 0u;
          const uint32_t d = tb + C::kS16 + hoff * kHalf;
          const uint64_t dk = dk16_0 + slot_off + hoff * (kHalf * 128 / 16);
          const uint32_t id = halves16 == 3u ? id16_full : id16_half;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint64_t o = (ks >> 2) * (kBM * 128 / 16) + k_step(ks);
            const uint64_t ok_ = (ks >> 2) * (kBN * 128 / 16) + k_step(ks);
            mma_f16_ss(d, dq + o, dk + ok_, id, ks > 0 ? 1u : 0u);
          }
        }
        if (halves8) {
          const uint64_t dq = t ? dq8_1 : dq8_0;
          const uint32_t hoff = (halves8 == 2u) ? 1u : 0u;
          const uint32_t d = tb + C::kS8 + hoff * kHalf;
          const uint64_t ring_off =
              QF ? static_cast<uint64_t>(n & 1) * (C::kK8Bytes / 16) : slot_off;
          const uint64_t dk = dk8_0 + ring_off + hoff * (kHalf * D / 16);
          const uint32_t id = halves8 == 3u ? id8_full : id8_half;
#pragma unroll
          for (int ks = 0; ks < D / 32; ++ks)
            mma_i8_ss(d, dq + ks * 2, dk + ks * 2, id, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars[C::kBarS + t]);
        return true;
      };
      // O_t += P_t(n) V(n), P_t(n) read from TMEM.
      auto issue_pv = [&](int t, int n) -> bool {
        if (n > (t ? nl1 : nl0)) return true;
        const int s = n % C::kVStages;
        if (!mbar_wait(&bars[C::kBarP + t], n & 1, abort_flag)) return false;
        // INT8 cache: the converters' fp16 V (they waited for the TMA)
        if (!mbar_wait(&bars[(KV8 ? C::kBarVConv : C::kBarV) + s],
                       (n / C::kVStages) & 1, abort_flag))
          return false;
        tc_fence_after();
        const uint64_t dv = dv_0 + static_cast<uint64_t>(s) * kVSlotStep;
        const uint32_t tb = tmem + t * C::kTileCols;
        const uint32_t acc0 = n > 0 ? 1u : 0u;
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks)
          mma_f16_ts(tb + C::kOCol, tb + C::p_col(ks >> 2) + (ks & 3) * 8,
                     dv + ks * (16 * 128 / 16), idesc_pv, ks > 0 ? 1u : acc0);
        mma_commit(&bars[C::kBarO + t]);
        return true;
      };

      // S is single-buffered per query tile: Q K^T of tile n+1 follows the
      // P V that reads P of tile n.  A K slot frees when every query tile's
      // Q K^T of it completed, a V slot when every P V did.
      for (int t = 0; t < kQT && ok; ++t) ok = issue_qk(t, 0);
      if (ok) {
        mma_commit(&bars[C::kBarKEmpty + 0]);
        if (QF) mma_commit(&bars[C::kBarK8Empty + 0]);
      }
      for (int n = 0; n <= n_end && ok; ++n) {
        for (int t = 0; t < kQT && ok; ++t) {
          ok = issue_pv(t, n);
          if (ok) ok = issue_qk(t, n + 1);
        }
        if (ok) {
          mma_commit(&bars[C::kBarVEmpty + n % C::kVStages]);
          if (n + 1 <= n_end) {
            mma_commit(&bars[C::kBarKEmpty + (n + 1) % C::kKStages]);
            if (QF) mma_commit(&bars[C::kBarK8Empty + ((n + 1) & 1)]);
          }
        }
      }
      if (!ok) fail();
      // Drain: every MMA issued above has finished once this completes.
      mma_commit(&bars[C::kBarDrain]);
      mbar_wait(&bars[C::kBarDrain], 0, nullptr);
    }
    __syncwarp();
  } else if (warp >= kWarpConv) {
    // =================== INT8 KV cache converters (2 warps) ===================
    // Per key tile: K8 -> fp16 K (exact; only when some query tile routes
    // part of the tile to FP16) and V8 -> fp16 v8 * v_scale.  Each thread
    // converts whole key rows (rows ct and ct + 64), reading a row before
    // writing it, which makes the in-place V conversion safe.
    if (KV8) {
      const int ct = (warp - kWarpConv) * 32 + lane;
      const float* vscale =
          p.v_scale + (static_cast<size_t>(hk) * p.batch + b) * p.nbk;
      constexpr uint32_t k8_swz = D == 128 ? 7u : 3u;
      bool ok = true;
      for (int n = 0; n <= n_end && ok; ++n) {
        const int ks = n % C::kKStages;
        const bool got_k = mbar_wait(&bars[C::kBarK + ks],
                                     (n / C::kKStages) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, got_k)) {
          ok = false;
          break;
        }
        uint32_t kinds = 0;
        for (int t = 0; t < kQT; ++t)
          kinds |= kinds_of(t, n, 0) | kinds_of(t, n, 1);
        if (kinds & kKindF16) {
          uint8_t* kslot_p = kslot(ks);
#pragma unroll 1
          for (int rr = ct; rr < kBN; rr += 64)
            convert_row<D, false, kBN * 128>(kslot_p + C::kK8Off, k8_swz, kslot_p, rr,
                                  __float2half2_rn(1.0f));
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[C::kBarKConv + ks]);

        const int vs = n % C::kVStages;
        const bool got_v = mbar_wait(&bars[C::kBarV + vs],
                                     (n / C::kVStages) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, got_v)) {
          ok = false;
          break;
        }
        uint8_t* vslot_p = vslot(vs);
#pragma unroll 1
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
    if (QF) {
      // =================== on-chip quantisation (2 warps) ===================
      // Q8 of each query tile once (from Q in shared memory), then K8 of
      // each key tile that some row routes to INT8, with the quantiser's
      // definition over the block's rows inside the sequence (a 128-row tile
      // is one 128-token block).  K rows are read from global memory (L2),
      // not from the K slot, into a two-slot K8 ring, so the converters run
      // up to two key tiles ahead of the MMAs instead of waiting for each
      // fp16 K tile to land.  Each thread quantises whole rows (ct and
      // ct + 64); the block max combines the two warps through shared memory.
      const int cw = warp - kWarpConv;
      const int ct = cw * 32 + lane;
      float* aux = reinterpret_cast<float*>(smem + C::kAuxOff);
      float* sq_s = aux;          // [2] Q scale of each query tile
      float* sk_ring = aux + 2;   // [kSkRing] K scale of key tile n % ring
      float* xmax = aux + 2 + C::kSkRing;  // [2 slots][2 warps]
      constexpr uint32_t i8_swz = D == 128 ? 7u : 3u;
      uint32_t xu = 0;  // max exchanges so far
      bool ok = true;
      auto block_max = [&](float v, bool& good) -> float {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
        float* slot = xmax + (xu & 1) * 2;
        if (lane == 0) slot[cw] = v;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[C::kBarCvX]);
        const bool got = mbar_wait(&bars[C::kBarCvX], xu & 1, abort_flag);
        good = __all_sync(0xffffffffu, got);
        const float other = slot[1 - cw];
        ++xu;
        return fmaxf(v, other);
      };
      const bool got_q = mbar_wait(&bars[C::kBarQ], 0, abort_flag);
      ok = __all_sync(0xffffffffu, got_q);
      for (int t = 0; t < kQT && ok; ++t) {
        const TileRoute R = rt(t);
        bool any8 = false;
        for (int n = 0; n <= R.n_last; ++n)
          any8 |= ((kinds_of(t, n, 0) | kinds_of(t, n, 1)) & kKindI8) != 0;
        float sq = 0.0f;
        if (any8) {
          const int row0 = row_base + t * kBM;
          float local = 0.0f;
          for (int rr = ct; rr < kBM; rr += 64)
            if (row0 + rr < len) local = fmaxf(local, row_absmax_f16<D>(sQ(t), rr));
          bool good = true;
          const float amax = block_max(local, good);
          if (!good) {
            ok = false;
            break;
          }
          sq = __fdiv_rn(amax, 127.0f);
          const float rcp = amax != 0.0f ? __frcp_rn(sq) : 0.0f;
          for (int rr = ct; rr < kBM; rr += 64)
            quant_row<D>(sQ(t), sQ8(t), i8_swz, rr, sq, rcp);
          fence_proxy_async_smem();
        }
        if (ct == 0) sq_s[t] = sq;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[C::kBarQConv + t]);
      }
      // K rows of this CTA's KV head: row j of the sequence at kg + j * kstr
      const __half* kg = reinterpret_cast<const __half*>(p.k) +
                         (static_cast<size_t>(start) * p.hkv + hk) * D;
      const size_t kstr = static_cast<size_t>(p.hkv) * D;
      uint8_t* k8ring = smem + C::kK8Ring0;
      for (int n = 0; n <= n_end && ok; ++n) {
        const int rs = n & 1;
        // ring slot rs is free once both query tiles' Q K^T of tile n - 2
        // completed
        if (n >= 2) {
          const bool got = mbar_wait(&bars[C::kBarK8Empty + rs],
                                     ((n >> 1) - 1) & 1, abort_flag);
          if (!__all_sync(0xffffffffu, got)) {
            ok = false;
            break;
          }
        }
        const uint32_t code = qk_code(0, n) | (qk_code(1, n) << 4);
        float sk = 0.0f;
        if (code & 0xccu) {
          float local = 0.0f;
          for (int rr = ct; rr < kBN; rr += 64)
            if (n * kBN + rr < len)
              local = fmaxf(local,
                            row_absmax_global<D>(kg + (n * kBN + rr) * kstr));
          bool good = true;
          const float amax = block_max(local, good);
          if (!good) {
            ok = false;
            break;
          }
          sk = __fdiv_rn(amax, 127.0f);
          const float rcp = amax != 0.0f ? __frcp_rn(sk) : 0.0f;
          uint8_t* k8 = k8ring + rs * C::kK8Bytes;
          for (int rr = ct; rr < kBN; rr += 64)
            quant_row_global<D>(
                n * kBN + rr < len ? kg + (n * kBN + rr) * kstr : nullptr, k8,
                i8_swz, rr, sk, rcp);
          fence_proxy_async_smem();
        }
        if (ct == 0) sk_ring[n % C::kSkRing] = sk;
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars[C::kBarK8Full + rs]);
          mbar_arrive(&bars[C::kBarSK + n % C::kSkRing]);
        }
      }
      if (!ok) fail();
    }
  } else {
    // =================== softmax warps 0-15 ===================
    // Warpgroups 2t and 2t+1 serve query tile t: thread = score row = TMEM
    // lane, warpgroup 2t + hw takes keys 64*hw .. 64*hw+63 of every row.  The
    // two tiles' warpgroups run at the same time, one warp of each on every
    // SM sub-partition, so one tile's latencies hide behind the other's
    // arithmetic.  A tile's row max is combined by its two warpgroups
    // through shared memory; each keeps the sum of its own keys and the two
    // are added once, at the end.
    const int wg = warp >> 2;
    const int t = wg >> 1;    // query tile
    const int hw = wg & 1;    // key half
    const int r = threadIdx.x & 127;
    const int c0 = hw * kHalf;  // first key of this thread inside a key tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    bool ok = true;
    if (t < kQT) {
      const TileRoute R = rt(t);
      const int r_local = row_base + t * kBM + r;
      const int rh = DUAL ? (r >> 6) : 0;  // routing row half
      const uint64_t my_w = rh ? R.w1 : R.w0;
      const int my_nl = rh ? R.nl1 : R.nl0;
      const int key_lim = min(r_local, len - 1);  // keys j <= key_lim legal
      const uint32_t lane_addr = tmem + t * C::kTileCols + lane_off;
      const float* kscale =
          (routed || KV8)
              ? p.k_scale + (static_cast<size_t>(hk) * p.batch + b) * p.nbk
              : nullptr;
      // K scale of this thread's 64 keys; the next key tile's is fetched
      // while the current one is processed.
      auto ksc = [&](int n) {
        const int blk = (n * kBN + c0) / p.quant_block_k;
        return kscale[min(blk, p.nbk - 1)];
      };
      float sk_next =
          ((routed || KV8) && !QF && R.n_last >= 0) ? ksc(0) : 0.0f;
      // On-chip quantisation: the converters' scales in shared memory.
      const float* aux = reinterpret_cast<const float*>(smem + C::kAuxOff);
      // INT8 KV cache: the V scale's mantissa factor f in [1, 2) of this
      // thread's 64 keys (the converters put its power of two into V).
      const float* vscale =
          KV8 ? p.v_scale + (static_cast<size_t>(hk) * p.batch + b) * p.nbk
              : nullptr;
      auto vfrac = [&](int n) {
        const int blk = (n * kBN + c0) / p.quant_block_k;
        const float sv = vscale[min(blk, p.nbk - 1)];
        int e = 0;
        frexpf(sv, &e);
        return sv > 0.0f ? ldexpf(sv, 1 - e) : 1.0f;
      };
      float fv_next = (KV8 && R.n_last >= 0) ? vfrac(0) : 1.0f;
      // softmax scale (log2 units) times the Q block scale of this row: the
      // INT8 path's S c = (Q8 K8^T) sq sk scale log2(e)
      float cq =
          (routed && !QF)
              ? p.scale_log2 *
                    p.q_scale[(static_cast<size_t>(h) * p.batch + b) * p.nbq +
                              key_lim / p.quant_block_q]
              : 0.0f;
      if (QF && routed && R.n_last >= 0) {
        const bool got = mbar_wait(&bars[C::kBarQConv + t], 0, abort_flag);
        ok = __all_sync(0xffffffffu, got);
        cq = p.scale_log2 * aux[t];
      }
      // running max and (this warpgroup's) sum of the row
      float m_run = -CUDART_INF_F, l_run = 0.0f;
      uint32_t u = 0;  // exchanges so far: slot and parity
      float* red_t = red + t * 512;
      uint64_t* bar_red = &bars[C::kBarRed + 2 * t];
      // Combine a per-row value with the other warpgroup's (max or sum).
      auto exchange = [&](float v, bool& good) -> float {
        float* slot = red_t + (u & 1) * 256;
        slot[hw * 128 + r] = v;
        __syncwarp();  // orders the lanes' stores before lane 0's release
        if (lane == 0) mbar_arrive(&bar_red[u & 1]);
        const bool got = mbar_wait(&bar_red[u & 1], (u >> 1) & 1, abort_flag);
        good = __all_sync(0xffffffffu, got);
        const float other = slot[(1 - hw) * 128 + r];
        ++u;
        return other;
      };

      for (int n = 0; n <= R.n_last && ok; ++n) {
        float sk = sk_next;
        if ((routed || KV8) && !QF && n < R.n_last) sk_next = ksc(n + 1);
        if (QF && routed) {
          const int slot = n % C::kSkRing;
          const bool got = mbar_wait(&bars[C::kBarSK + slot],
                                     (n / C::kSkRing) & 1, abort_flag);
          if (!__all_sync(0xffffffffu, got)) {
            ok = false;
            break;
          }
          sk = aux[2 + slot];
        }
        const float fv = fv_next;
        if (KV8 && n < R.n_last) fv_next = vfrac(n + 1);
        // Exits stay warp-uniform: the tcgen05.ld/st below are .sync.aligned.
        const bool got_s = mbar_wait(&bars[C::kBarS + t], n & 1, abort_flag);
        if (!__all_sync(0xffffffffu, got_s)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // Path of this thread's 64 keys for its routing row half.  Keys past
        // every row of the tile: the MMA wrote the first half's path there
        // (values masked below either way).
        const int n64 = 2 * n + hw;
        const int nb = (!DUAL && n64 > my_nl) ? 2 * n : n64;
        const bool i8 =
            (nb <= my_nl) && (((my_w >> (nb / tpb)) & 1ull) != 0);
        // FP16 keys of the INT8 cache are k8 exactly: their scale joins c.
        const float c = i8 ? cq * sk : (KV8 ? p.scale_log2 * sk : p.scale_log2);
        const uint32_t scol = lane_addr + (i8 ? C::kS8 : C::kS16) + c0;
        const int hl = key_lim - n * kBN - c0;  // legal columns: j <= hl
        float mx;
        {  // pass 1: the 64 scores only live for the row max
          uint32_t sv[kHalf];
          tmem_ld32(scol, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
          tmem_ld32(scol + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
          tmem_ld_wait();
          if (p.qk_dump && r_local < len && i8 && n64 <= my_nl) {
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
          const bool fullh = hl >= kHalf - 1;
          mx = i8 ? (fullh ? max64<true, false>(sv, hl)
                           : max64<true, true>(sv, hl))
                  : (fullh ? max64<false, false>(sv, hl)
                           : max64<false, true>(sv, hl));
        }
        const float m_half = (mx == -CUDART_INF_F) ? -CUDART_INF_F : mx * c;
        bool good = true;
        const float m_tile = fmaxf(m_half, exchange(m_half, good));
        if (!good) {
          ok = false;
          break;
        }
        // Lazy rescaling: keep the old max unless the tile exceeds it by
        // more than 2^threshold, so P <= 2^threshold stays in fp16 range.
        // (the fp16-accumulator study keeps P <= 1: fp16 O has no headroom)
        const bool need =
            m_tile > m_run + (p.pv_f16_acc ? 0.0f : kRescaleThreshold);
        const float m_old = m_run;
        if (need) {
          l_run *= ex2_approx(m_run - m_tile);
          m_run = m_tile;
        }
        // P = 2^(S c - m) of this thread's 64 keys as fp16 pairs over the S
        // columns it has just read (key 2i in the low half of column i).
        float2 ps0 = make_float2(0.f, 0.f), ps1 = ps0, ps2 = ps0, ps3 = ps0;
        float unused_max = 0.0f;
        // INT8 KV cache: P f = 2^(S c - m + log2 f) goes to the P V product
        // (<= 2^9, fp16-safe); the row sum divides f out again.
        const float m_exp = KV8 ? m_run - __log2f(fv) : m_run;
#pragma unroll
        for (int q = 0; q < 2; ++q) {  // pass 2: reload 32 scores at a time
          uint32_t sq32[32];
          tmem_ld32(scol + 32 * q, sq32);
          tmem_ld_wait();
          uint32_t pk[16];
          const int hq = hl - 32 * q;
          const bool fullq = hq >= 31;
          if (i8) {
            if (fullq) exp32<true, false, false>(sq32, c, m_exp, hq, pk, ps0, ps1, ps2, ps3, unused_max);
            else exp32<true, true, false>(sq32, c, m_exp, hq, pk, ps0, ps1, ps2, ps3, unused_max);
          } else {
            if (fullq) exp32<false, false, false>(sq32, c, m_exp, hq, pk, ps0, ps1, ps2, ps3, unused_max);
            else exp32<false, true, false>(sq32, c, m_exp, hq, pk, ps0, ps1, ps2, ps3, unused_max);
          }
          tmem_st16(lane_addr + C::p_col(hw) + 16 * q, pk);
        }
        if (n > 0 && __any_sync(0xffffffffu, need)) {
          // S_t(n) is ready, so P V_t(n-1) completed (the MMA thread issues
          // Q K^T_t(n) after it): O_t can be rescaled now.  Each warpgroup
          // rescales half of O's columns.
          const float alpha = need ? ex2_approx(m_old - m_tile) : 1.0f;
          const int o0 = hw * (D / 2);
#pragma unroll
          for (int oc = 0; oc < D / 2; oc += 32) {
            uint32_t o[32];
            tmem_ld32(lane_addr + C::kOCol + o0 + oc, o);
            tmem_ld_wait();
            if (p.pv_f16_acc) {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                o[j] = __half_as_ushort(__float2half_rn(
                    __half2float(__ushort_as_half(static_cast<uint16_t>(o[j]))) *
                    alpha));
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
            }
            tmem_st32(lane_addr + C::kOCol + o0 + oc, o);
          }
        }
        const float2 s4 = __fadd2_rn(__fadd2_rn(ps0, ps1), __fadd2_rn(ps2, ps3));
        l_run += KV8 ? (s4.x + s4.y) / fv : s4.x + s4.y;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[C::kBarP + t]);
      }

      // Epilogue: O / l with both warpgroups' sums; each warpgroup stores
      // half of O's columns.
      if (ok && R.n_last >= 0) {
        const bool got_last =
            mbar_wait(&bars[C::kBarO + t], R.n_last & 1, abort_flag);
        ok = __all_sync(0xffffffffu, got_last);
        if (ok) {
          tc_fence_after();
          bool good = true;
          const float l_tot = l_run + exchange(l_run, good);
          ok = good;
          if (ok) {
            const bool valid = r_local < len;
            const float inv_l = 1.0f / l_tot;
            const int o0 = hw * (D / 2);
            // A tile whose 128 rows all lie in the sequence leaves through
            // one bulk store from shared memory (its Q buffer is free now);
            // a partial tile stores its valid rows directly.
            const bool full = row_base + t * kBM + kBM <= len;
            uint8_t* stage = sQ(t);
            uint16_t* orow =
                p.out + (static_cast<size_t>(start + r_local) * p.hq + h) * D +
                o0;
#pragma unroll
            for (int oc = 0; oc < D / 2; oc += 32) {
              uint32_t o[32];
              tmem_ld32(lane_addr + C::kOCol + o0 + oc, o);
              tmem_ld_wait();
              if (p.pv_f16_acc) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  o[j] = __float_as_uint(__half2float(
                      __ushort_as_half(static_cast<uint16_t>(o[j]))));
              }
              uint32_t hv[16];
#pragma unroll
              for (int j = 0; j < 16; ++j)
                hv[j] = pack_half2(__uint_as_float(o[2 * j]) * inv_l,
                                   __uint_as_float(o[2 * j + 1]) * inv_l);
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                const uint4 val = make_uint4(hv[4 * v], hv[4 * v + 1],
                                             hv[4 * v + 2], hv[4 * v + 3]);
                if (full) {
                  // column o0 + oc + 8v: chunk (o0 + oc) / 64, 16-byte
                  // unit ((o0 + oc) % 64) / 8 + v of row r, 128B swizzle
                  const int col = o0 + oc + 8 * v;
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
              if (threadIdx.x == t * 256) {
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
            if (p.lse && valid && hw == 0)
              p.lse[static_cast<size_t>(h) * p.total_tokens + start + r_local] =
                  (m_run + __log2f(l_tot)) * 0.69314718055994530942f;
          }
        }
      }
    }
    if (!ok) fail();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) tmem_dealloc(tmem, C::kTmemCols);
}

template <int D, bool DUAL, int MODE>
cudaError_t launch_one(const AttnParams& p, cudaStream_t stream) {
  using C = Cfg<D, DUAL, MODE>;
  auto kern = attn_fwd_kernel<D, DUAL, MODE>;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const int groups = (p.max_seqlen + C::kQT * kBM - 1) / (C::kQT * kBM);
  dim3 grid(p.hq, groups, p.batch);
  kern<<<grid, threads_of(MODE), C::kSmem, stream>>>(p);
  return cudaGetLastError();
}

template <int D, int MODE>
cudaError_t launch_dm(const AttnParams& p, const AttnLaunchShape& s,
                      cudaStream_t stream) {
  return s.dual ? launch_one<D, true, MODE>(p, stream)
                : launch_one<D, false, MODE>(p, stream);
}

template <int D>
cudaError_t launch_d(const AttnParams& p, const AttnLaunchShape& s,
                     cudaStream_t stream) {
  if (s.mode == kModeKV8) return launch_dm<D, kModeKV8>(p, s, stream);
  if (s.mode == kModeOnChip) return launch_dm<D, kModeOnChip>(p, s, stream);
  return launch_dm<D, kModeGiven>(p, s, stream);
}

template <int D, int MODE>
int smem_dm(const AttnLaunchShape& s) {
  return s.dual ? Cfg<D, true, MODE>::kSmem : Cfg<D, false, MODE>::kSmem;
}

template <int D>
int smem_d(const AttnLaunchShape& s) {
  if (s.mode == kModeKV8) return smem_dm<D, kModeKV8>(s);
  if (s.mode == kModeOnChip) return smem_dm<D, kModeOnChip>(s);
  return smem_dm<D, kModeGiven>(s);
}

}  // namespace

cudaError_t launch_attn_prefill(const AttnParams& p, const AttnLaunchShape& s,
                                cudaStream_t stream) {
  if (s.head_dim == 128) return launch_d<128>(p, s, stream);
  if (s.head_dim == 64) return launch_d<64>(p, s, stream);
  return cudaErrorInvalidValue;
}

int attn_smem_bytes(const AttnLaunchShape& s) {
  if (s.head_dim == 128) return smem_d<128>(s);
  if (s.head_dim == 64) return smem_d<64>(s);
  return -1;
}

}  // namespace tilemix
