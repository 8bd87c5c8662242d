/*
 * tilemix.h - C ABI of the tile-routed FP16/INT8 causal prefill attention
 * library for NVIDIA B200 (sm_100a).
 *
 * The operation follows "TileMix: Tile-Centric Mixed-Precision Attention for
 * LLM Inference Acceleration" (arXiv 2608.17336) as summarised on its public
 * pages.  The causal score matrix of every sequence is cut into BM x BN score
 * tiles; one 64-bit routing word per (sequence, KV head, query-tile row)
 * carries one bit per group of g adjacent key tiles; a legal tile group whose
 * bit is 1 computes its scores as Q8 K8^T on INT8 tensor cores with INT32
 * accumulation, rescaled by the two block scales, and one whose bit is 0
 * computes them as Q K^T in FP16; both feed the same online-softmax state and
 * the FP16 P V product.
 *
 * Conventions shared by every call:
 *  - Pointers marked "dev" are CUDA device pointers, owned by the caller,
 *    which must keep them alive until the stream work completes.  The
 *    library allocates nothing, never synchronises the device or the stream,
 *    and copies nothing between host and device.
 *  - Every call is asynchronous on `stream` (NULL = the legacy default
 *    stream) and returns after enqueueing its kernels.
 *  - Token-major, unpadded layout: a tensor "[T, H, d]" holds the T = sum of
 *    all sequence lengths tokens back to back, each token's H heads back to
 *    back, each head's d channels contiguous.  Sequence b spans tokens
 *    [cu_seqlens[b], cu_seqlens[b+1]).
 *  - Argument errors are detected on the host before anything is launched;
 *    the call then returns a status other than TILEMIX_OK, launches nothing,
 *    and tilemix_last_error() describes the problem.
 *  - Problems only the device can see (a non-monotone cu_seqlens, a length
 *    above max_seqlen, a head_map entry out of range, a pipeline wait that
 *    ran past its time limit) are reported through the optional `status`
 *    word (dev int32): the first kernel to see one stores its
 *    tilemix_status code there (if the word is still 0) and its blocks
 *    return without touching the outputs they would have written; blocks
 *    of tilemix_attn_prefill that start while the word is nonzero return at
 *    once.  The caller zeroes the word before the call and reads it after
 *    the stream work completes.  Kernels never trap.
 *  - Inputs must be finite.  NaN or Inf input gives undefined output.
 */
#ifndef TILEMIX_H_
#define TILEMIX_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* tilemix_stream_t;

typedef enum {
  TILEMIX_OK = 0,
  TILEMIX_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size       */
  TILEMIX_ERR_UNSUPPORTED = 2,  /* valid but not built (d, tile shape ...) */
  TILEMIX_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed       */
  TILEMIX_ERR_TIMEOUT = 4,      /* device: a pipeline wait ran too long    */
  TILEMIX_ERR_BAD_SEQLENS = 5,  /* device: cu_seqlens or head_map invalid  */
  TILEMIX_ERR_NO_DEVICE = 6     /* current device is not sm_100            */
} tilemix_status;

enum { TILEMIX_KV_FP16 = 0, TILEMIX_KV_INT8 = 1 };

/* Ignore the routing words: every legal tile takes the FP16 path and the
 * INT8 operands (q8, q_scale, and k8, k_scale for TILEMIX_KV_FP16) may be
 * NULL.  This is the all-FP16 reference mode. */
#define TILEMIX_FLAG_FP16_ONLY 1u

/* On-the-fly quantisation (paperlayer summary, appendix C Quantization
 * Configuration: INT8 fragments generated only for routed groups, scales
 * computed and applied on chip).  The kernel quantises each Q tile and each
 * key tile that some row routes to INT8 itself, with the quantiser's exact
 * definition (one scale per 128-token block; needs quant_block_q =
 * quant_block_k = 128), so results equal a tilemix_quantize_blockwise call
 * followed by the quantize-once attention.  q8, q_scale, k8 and k_scale are
 * not read (may be NULL).  TILEMIX_KV_FP16 only. */
#define TILEMIX_FLAG_QUANT_ON_CHIP 2u

/* Test only: the kernel withholds the first V tile of every CTA, so the
 * consumers' bounded pipeline wait expires (after about 2 s): the call
 * reports TILEMIX_ERR_TIMEOUT in *status, writes no defined output, and the
 * context stays usable.  It exercises the timeout path; no fault, trap or
 * unbounded wait is involved.  Not for production calls. */
#define TILEMIX_FLAG_TEST_EXPIRE_WAIT 4u

/* Study only (paperlayer summary, appendix G Numerical Analysis: the
 * deviation of FP16 against FP32 accumulation): the P V product accumulates
 * O in fp16 in Tensor Memory (kind::f16 MMA with an F16 D format) instead
 * of fp32; the running max, the row sum and the final O / l stay fp32.
 * Results are NOT held to the output tolerance of the default mode; the
 * flag exists to measure how far fp16 accumulation moves the output. */
#define TILEMIX_FLAG_PV_F16_ACC 8u

/*
 * Blockwise symmetric INT8 quantisation ("quantize-once").
 * Pages: section 3 Preliminaries (blockwise quantization; INT8 tensor cores
 * with INT32 accumulation) and appendix C Quantization Configuration
 * (blockwise symmetric INT8 of Q and K, made once per attention call).
 *
 * For every sequence b, head h and block t of `block` consecutive tokens of
 * that sequence (blocks restart at each sequence start; the last block of a
 * sequence may be short):
 *   a = max |x| over the block's tokens and d channels,
 *   scale[h][b][t] = a / 127            (one IEEE fp32 division),
 *   x8 = clamp(round_half_even(x / scale), -127, 127) (IEEE fp32 division),
 *   a == 0 gives scale 0 and codes 0.
 * Blocks t >= ceil(len_b / block) of a shorter sequence get scale 0.
 *
 *   x          dev fp16 [T, heads, head_dim], 16-byte aligned
 *   cu_seqlens dev int32 [batch + 1], non-decreasing, cu_seqlens[0] = 0
 *   max_seqlen host int: >= every sequence length
 *   total_tokens host int: T = cu_seqlens[batch], the rows of x and x8
 *   head_dim   multiple of 8, <= 256; block in [1, 256], block*head_dim <= 32768
 *   x8         dev int8 [T, heads, head_dim], 16-byte aligned
 *   scale      dev fp32 [heads, batch, ceil(max_seqlen / block)]
 *   status     optional dev int32 (see above)
 */
tilemix_status tilemix_quantize_blockwise(
    const void* x, const int32_t* cu_seqlens, int batch, int max_seqlen,
    int total_tokens, int heads, int head_dim, int block, int8_t* x8,
    float* scale, int32_t* status, tilemix_stream_t stream);

/*
 * Q and K of one attention call quantised in one launch.
 * Pages: appendix C Quantization Configuration (Q and K quantised blockwise
 * and symmetrically once per call) and section 3 Preliminaries.
 * The results are exactly those of tilemix_quantize_blockwise(q, ..., hq,
 * head_dim, block_q, q8, q_scale) followed by tilemix_quantize_blockwise(k,
 * ..., hkv, head_dim, block_k, k8, k_scale); one grid covers the blocks of
 * both tensors.
 *
 *   q, k        dev fp16 [T, hq, head_dim] and [T, hkv, head_dim], 16-byte aligned
 *   q8, k8      dev int8, same shapes, 16-byte aligned
 *   q_scale     dev fp32 [hq, batch, ceil(max_seqlen / block_q)]
 *   k_scale     dev fp32 [hkv, batch, ceil(max_seqlen / block_k)]
 *   block_q, block_k  as `block` above; hq + hkv <= 65535
 * Errors as for tilemix_quantize_blockwise; nothing is launched when an
 * argument is rejected.
 */
tilemix_status tilemix_quantize_blockwise_qk(
    const void* q, const void* k, const int32_t* cu_seqlens, int batch,
    int max_seqlen, int total_tokens, int hq, int hkv, int head_dim,
    int block_q, int block_k, int8_t* q8, float* q_scale, int8_t* k8,
    float* k_scale, int32_t* status, tilemix_stream_t stream);

/*
 * Pack per-group routing bytes into 64-bit routing words.
 * Pages: section 3 Preliminaries (packed 64-bit masks, bit floor(n/g) of the
 * word of a query-tile row selects the path of key tile n), section 4
 * (routing map indexed by KV head, query-tile row and key-tile group), and
 * the gist.science technical summary (lookup R = (b >> g_j) & 1).
 *
 * Output bit j of word [b][hk][m] is (route[b][hk][m][j] != 0) for every
 * group j that holds a legal (causal, in-sequence) query/key pair of
 * query-tile row m; every other bit is 0 (junk in illegal groups is
 * cleared).  1 = INT8, 0 = FP16.
 *
 *   route      dev uint8 [batch, hkv, Tm_max, 64], Tm_max = ceil(max_seqlen/block_m)
 *   block_m, block_n  score-tile shape the words will be read with
 *   group      g >= 1 with ceil(ceil(max_seqlen / block_n) / g) <= 64
 *   mask       dev uint64 [batch, hkv, Tm_max], 8-byte aligned
 */
tilemix_status tilemix_pack_mask(
    const uint8_t* route, const int32_t* cu_seqlens, int batch,
    int max_seqlen, int hkv, int block_m, int block_n, int group,
    uint64_t* mask, int32_t* status, tilemix_stream_t stream);

/*
 * Static routing templates: route bytes (1 = INT8, 0 = FP16) for a named
 * spatial layout at a given INT8 coverage, ready for tilemix_pack_mask.
 * Pages: paperlayer summary appendix B Precision Layouts (uniform All INT8
 * and All FP16 references; Band, Global, Row-Random, Aligned Sparse,
 * BigBird and SpTrans templates; 25/50/75% = INT8 share of legal tile
 * groups) and Limitations (static templates give deterministic policies;
 * the kernel consumes any static or adaptive policy).  The pages give the
 * names only; the definitions below are this library's readings.
 *
 * Per query-tile row (b, hk, m) with G legal groups (the groups holding a
 * causal in-sequence pair; group j covers key tiles g*j .. g*j+g-1) and
 * distance d = G - 1 - j from the diagonal group:
 *   k_int8 = (int8_permille * G + 500) / 1000 (integer division),
 *   FP16 goes to the G - k_int8 groups with the largest key
 *   (priority(j) << 32) | h32(j), ties to the smaller j, where h32 is the
 *   high half of splitmix64 (Steele, Lea and Flood 2014) of
 *   seed + (c + 1) * 0x9E3779B97F4A7C15 with counter
 *   c = ((b * hkv + hk) * Tm_max + m) * 64 + j:
 *     ALL_FP16     every legal group FP16 (int8_permille ignored)
 *     ALL_INT8     every legal group INT8 (int8_permille ignored)
 *     BAND         priority 63 - d     (FP16 band along the diagonal)
 *     GLOBAL       priority 63 - j     (FP16 on the first key groups)
 *     ROW_RANDOM   priority 0          (a random subset of each row)
 *     ALIGNED      priority 1 when j % 4 == 0, else 0
 *     BIGBIRD      priority 1 when j == 0 or d <= 1, else 0
 *     SPTRANS      priority 2 when d <= 1, 1 when j % 4 == 3, else 0
 * Bytes of illegal groups and of rows past a sequence are 0.
 *
 *   layout         TILEMIX_LAYOUT_*
 *   int8_permille  INT8 share of each row's legal groups, in [0, 1000]
 *   route          dev uint8 [batch, hkv, Tm_max, 64] (written entirely)
 *   other arguments as for tilemix_pack_mask
 */
enum {
  TILEMIX_LAYOUT_ALL_FP16 = 0,
  TILEMIX_LAYOUT_ALL_INT8 = 1,
  TILEMIX_LAYOUT_BAND = 2,
  TILEMIX_LAYOUT_GLOBAL = 3,
  TILEMIX_LAYOUT_ROW_RANDOM = 4,
  TILEMIX_LAYOUT_ALIGNED = 5,
  TILEMIX_LAYOUT_BIGBIRD = 6,
  TILEMIX_LAYOUT_SPTRANS = 7
};

tilemix_status tilemix_route_template(
    int layout, int int8_permille, uint64_t seed, const int32_t* cu_seqlens,
    int batch, int max_seqlen, int hkv, int block_m, int block_n, int group,
    uint8_t* route, int32_t* status, tilemix_stream_t stream);

/*
 * Adaptive routing from a cheap score statistic, run on the device before
 * the attention call.  Pages: paperlayer summary, Limitations (the kernel
 * interface accepts static or adaptive routing policies) and appendix G.5
 * (routing that keeps high-mass attention blocks in FP16 protects accuracy).
 * The pages define no statistic; this library's reading:
 *
 * For query-tile row m of sequence b and KV head hk, with G legal groups,
 *   Sq[c]   = sum over the row's in-sequence query rows i and the query
 *             heads h of hk of X(q[i][h][c]),
 *   Sk_j[c] = sum over the in-sequence keys of group j (key tiles
 *             g*j .. g*j+g-1) of X(k[key][hk][c]),
 *   I_j     = sum_c Sq[c] * Sk_j[c]  = 2^48 x the sum of all raw logits
 *             q.k between the row's queries (over hk's heads) and the
 *             group's keys,
 * where X(v) = v * 2^24 is the exact integer value of an fp16 number; every
 * sum is exact (64-bit for Sq, Sk; 128-bit for I), so the ranking does not
 * depend on summation order.  k_int8 = (int8_permille * G + 500) / 1000; the
 * G - k_int8 groups with the largest I_j stay FP16 (ties to the smaller j),
 * the rest INT8.  Output: route bytes as tilemix_route_template, and / or
 * the routing words the attention call reads.
 *
 *   q, k           dev fp16 [T, hq, d] / [T, hkv, d], 16-byte aligned;
 *                  d a multiple of 8 in [8, 256]
 *   head_map       optional dev int32 [hq] (NULL: contiguous groups of
 *                  hq / hkv query heads)
 *   workspace      dev scratch of at least
 *                  tilemix_route_adaptive_workspace_bytes() bytes (8 * d *
 *                  batch * hkv * (Tm_max + 64)), 16-byte aligned, owned by
 *                  the caller; overwritten; must not be shared with another
 *                  call that may run at the same time
 *   route          optional dev uint8 [batch, hkv, Tm_max, 64], 16-byte
 *                  aligned; bytes past a row's G legal groups and rows past
 *                  a sequence's end are written 0
 *   mask           optional dev uint64 [batch, hkv, Tm_max], 8-byte aligned:
 *                  the same decisions as packed routing words, equal to
 *                  tilemix_pack_mask of `route` (at least one of route and
 *                  mask is given)
 *
 * Errors: INVALID_ARG for null or misaligned pointers, bad sizes, a
 * permille outside [0, 1000], more than 64 groups or a short workspace;
 * UNSUPPORTED for tiles so large that the exact integer arithmetic could
 * overflow: with rows = block_m * query heads per KV head (hq with a
 * head_map) and keys = g * block_n, it needs rows, keys < 2^15, rows * d and
 * keys * d < 2^22, and rows * keys * d < 2^47.  Device side (status word): BAD_SEQLENS for
 * cu_seqlens outside [0, total_tokens] or above max_seqlen, or a head_map
 * entry outside [0, hkv).  The rows of such a sequence (with a bad head_map
 * entry: every row of the call) are not ranked; their route bytes and
 * routing words are written as 0.
 * Asynchronous on `stream`; allocates nothing.  The workspace query returns
 * 0 for negative or zero sizes.
 */
size_t tilemix_route_adaptive_workspace_bytes(int batch, int max_seqlen,
                                              int hkv, int head_dim,
                                              int block_m);

tilemix_status tilemix_route_adaptive(
    const void* q, const void* k, const int32_t* cu_seqlens, int batch,
    int max_seqlen, int total_tokens, int hq, int hkv, int head_dim,
    const int32_t* head_map, int block_m, int block_n, int group,
    int int8_permille, void* workspace, size_t workspace_bytes,
    uint8_t* route, uint64_t* mask, int32_t* status, tilemix_stream_t stream);

/*
 * tilemix_route_adaptive without a caller workspace, for callers that cannot
 * allocate device memory themselves: the same checks, the same kernels and
 * the same output, with the scratch taken from one static device array of
 * TILEMIX_ROUTE_ADAPTIVE_STATIC_BYTES per device.  The array is reserved
 * when the library's device code loads on that device, which with CUDA's
 * lazy module loading happens on the first call of a library kernel there:
 * make that first call outside any stream capture.  The call itself
 * allocates nothing; it looks the array's address up in the current context
 * each time.  No counterpart in the TileMix pages: an interface convenience
 * of this library.
 *
 * Errors: as tilemix_route_adaptive, and INVALID_ARG when the call would
 * need more than TILEMIX_ROUTE_ADAPTIVE_STATIC_BYTES of scratch
 * (tilemix_route_adaptive_workspace_bytes() says how much).
 *
 * Races: every call on a device shares the one scratch array.  Two calls
 * whose work can overlap on the device (different streams without an event
 * between them, different host threads, concurrent graph replays) overwrite
 * each other's statistics and may write wrong routing without any error.
 * Order such calls on one stream or with events; calls in one stream are
 * safe.
 */
#define TILEMIX_ROUTE_ADAPTIVE_STATIC_BYTES (32u << 20)

tilemix_status tilemix_route_adaptive_noalloc(
    const void* q, const void* k, const int32_t* cu_seqlens, int batch,
    int max_seqlen, int total_tokens, int hq, int hkv, int head_dim,
    const int32_t* head_map, int block_m, int block_n, int group,
    int int8_permille, uint8_t* route, uint64_t* mask, int32_t* status,
    tilemix_stream_t stream);


/*
 * Arguments of tilemix_attn_prefill.  Zero-initialise, set struct_size =
 * sizeof(tilemix_attn_params), then fill the fields.
 */
typedef struct {
  uint32_t struct_size;
  int kv_format;        /* TILEMIX_KV_FP16 or TILEMIX_KV_INT8 (INT8 cache)  */
  uint32_t flags;       /* TILEMIX_FLAG_*                                    */

  /* Q: fp16 [T, hq, d]; Q8: int8 [T, hq, d]; q_scale: fp32
   * [hq, batch, ceil(max_seqlen / quant_block_q)] (tilemix_quantize_blockwise
   * output).  All 16-byte aligned. */
  const void* q;
  const int8_t* q8;
  const float* q_scale;
  /* TILEMIX_KV_FP16: k, v fp16 [T, hkv, d]; k8 + k_scale (as for Q, block
   * quant_block_k) for INT8-routed groups.
   * TILEMIX_KV_INT8: k8, v8 int8 [T, hkv, d] with k_scale, v_scale fp32
   * [hkv, batch, ceil(max_seqlen / quant_block_k)]; k and v unused.  FP16
   * groups then use K = k8 * k_scale exactly; V = v8 * v_scale always. */
  const void* k;
  const int8_t* k8;
  const float* k_scale;
  const void* v;
  const int8_t* v8;
  const float* v_scale;

  const int32_t* cu_seqlens; /* dev int32 [batch + 1]                      */
  int batch;
  int max_seqlen;            /* host: >= every sequence length              */
  int total_tokens;          /* host: T = cu_seqlens[batch]; the kernels
                                never address a token row at or past T    */
  int hq, hkv, head_dim;     /* head_dim in {64, 128}                       */
  /* dev int32 [hq]: KV head of each query head (query heads mapped to one
   * KV head share its K, V and routing words).  NULL: contiguous groups,
   * KV head = h / (hq / hkv), which needs hq % hkv == 0. */
  const int32_t* head_map;

  /* Routing words from tilemix_pack_mask: dev uint64 [batch, hkv,
   * ceil(max_seqlen / block_m)].  Tile shape: block_m in {64, 128},
   * block_n in {64, 128} (block_m = 64 needs block_n = 64), group g >= 1
   * with ceil(ceil(max_seqlen / block_n) / g) <= 64.  Bits of illegal groups
   * are ignored. */
  const uint64_t* mask;
  int block_m, block_n, group;
  /* Quantisation block lengths in tokens: quant_block_q >= 1, quant_block_k
   * a multiple of block_n (one K scale per key tile). 0 = 128. */
  int quant_block_q, quant_block_k;
  float softmax_scale;       /* > 0; <= 0 means 1 / sqrt(head_dim)         */
  int causal;                /* must be 1                                   */

  void* out;                 /* dev fp16 [T, hq, d]                         */
  float* lse;                /* optional dev fp32 [hq, T]: natural-log LSE  */
  /* Optional debug output, dev int32 [batch, hq, Tm_max, Tn_max, block_m,
   * block_n] with Tn_max = ceil(max_seqlen / block_n): the raw INT32
   * accumulators of every INT8-routed legal tile, causally masked positions
   * included, written for the rows and keys inside the sequence.  Keys past
   * the last query row of the routing row (masked for all of its rows) may be
   * skipped in 64-key steps; every other entry is left untouched. */
  int32_t* qk_dump;
  int32_t* status;           /* optional dev int32, see above               */
} tilemix_attn_params;

/*
 * Causal tile-routed prefill attention (forward, GQA, unpadded varlen).
 * Pages: section 3 Preliminaries (S = QK^T, P = softmax(S), O = PV; online
 * softmax with row maxima and normalisers; FP16 and INT8 score tiles enter a
 * common domain before updating one maximum, normaliser and accumulator;
 * routing words and legality), section 4 (GQA and varlen routing),
 * appendices B-D (legality separate from routing; FP16 V/PV; quantize-once
 * operands; INT8 KV cache), ainews summary (shared online-softmax state).
 *
 * For query i and key j <= i of sequence b, query head h, KV head hk:
 *   route = bit floor(floor(j / block_n) / group) of
 *           mask[b][hk][floor(i / block_m)]            (1 = INT8)
 *   s_ij  = scale * sum_c q8_ic k8_jc * q_scale[h][b][i / qb] * k_scale[hk][b][j / kb]
 *           if route, else scale * sum_c q_ic k_jc
 *   out_i = sum_j softmax_j(s_i.) v_j ,  lse_i = ln sum_j exp(s_ij)
 * computed on sm_100a tensor cores (FP16 MMA with f32 accumulation, INT8
 * MMA with INT32 accumulation, FP16 P with f32 accumulation for P V).
 * Returns TILEMIX_ERR_NO_DEVICE when the current device is not sm_100.
 */
tilemix_status tilemix_attn_prefill(const tilemix_attn_params* params,
                                    tilemix_stream_t stream);

/* Static description of a status code. */
const char* tilemix_status_string(tilemix_status status);

/* Detail of the last error returned on the calling host thread ("" if none). */
const char* tilemix_last_error(void);

/* Library ABI version: (major << 16) | minor. */
uint32_t tilemix_version(void);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* TILEMIX_H_ */
