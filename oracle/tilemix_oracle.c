/*
 * CPU oracle for tile-routed FP16/INT8 causal prefill attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the timed
 * CPU baseline of the benchmark may load this file's library.  It shares no
 * code, header, table or helper with the CUDA path and never calls it.
 *
 * Written from the TileMix pages (arXiv 2608.17336):
 *  - quantiser: blockwise symmetric INT8 of Q and K, one scale per block of
 *    tokens per head ("TileMix: Tile-Centric Mixed-Precision Attention",
 *    paperlayer summary, section 3 Preliminaries and appendix C
 *    Quantization Configuration); scale = absmax / 127 in fp32, codes
 *    rounded half-to-even and clamped to +-127 (the convention fixed for
 *    this implementation);
 *  - routing words: one 64-bit word per (sequence, KV head, query-tile
 *    row); key tile n reads bit floor(n / g), 1 = INT8, 0 = FP16 (section 3
 *    Preliminaries; gist.science technical summary, "Enrutamiento por
 *    Mascara de Bits Compacta", formula R = (b >> g_j) & 1);
 *  - legality (causal and sequence boundary) is independent of routing
 *    (appendix B Precision Layouts);
 *  - scores: FP16 pairs use the fp16 Q and K; INT8 pairs use Q8 K8^T with
 *    integer accumulation, rescaled by the two block scales (section 3
 *    Preliminaries; gist.science "Ejecucion Heterogenea de Estado
 *    Compartido");
 *  - softmax and output: P = softmax(S), O = P V (section 3 Preliminaries),
 *    V always FP16 (appendix C), or an INT8 cache dequantised exactly.
 *
 * This oracle does not follow the fused kernel's structure: every row's
 * legal scores are materialised, then max, exp, sum and the weighted sum
 * of V are taken in fp64 in two passes.  Integer dots are exact in int64.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_GROUPS 2
#define ORACLE_ERR_ALLOC 3

/* IEEE 754 binary16 -> binary32, exact. */
static float half_bits_to_float(uint16_t h) {
  uint32_t sign = (uint32_t)(h >> 15) & 1u;
  uint32_t expo = (uint32_t)(h >> 10) & 0x1fu;
  uint32_t mant = (uint32_t)h & 0x3ffu;
  float mag;
  if (expo == 0) {
    mag = ldexpf((float)mant, -24); /* subnormal (or zero): mant * 2^-24 */
  } else if (expo == 31) {
    mag = mant ? NAN : INFINITY;
  } else {
    mag = ldexpf((float)(mant | 0x400u), (int)expo - 25);
  }
  return sign ? -mag : mag;
}

double oracle_half_to_double(uint16_t h) { return (double)half_bits_to_float(h); }

/* ------------------------------------------------------------------------ */
/* Quantiser                                                                */
/* ------------------------------------------------------------------------ */

/* x: fp16 bits [T, heads, d]; x8: int8 [T, heads, d];
 * scale: fp32 [heads, batch, nblk], nblk = ceil(max_seqlen / block).
 * Blocks restart at every sequence start.  Block entries past a sequence's
 * end are written as 0. */
int oracle_quantize_blockwise(const uint16_t* x, const int32_t* cu_seqlens,
                              int batch, int max_seqlen, int heads, int d,
                              int block, int8_t* x8, float* scale) {
  if (!x || !cu_seqlens || !x8 || !scale || batch < 0 || heads <= 0 ||
      d <= 0 || block <= 0 || max_seqlen < 0)
    return ORACLE_ERR_ARG;
  int nblk = (max_seqlen + block - 1) / block;
  for (int b = 0; b < batch; ++b) {
    int start = cu_seqlens[b];
    int len = cu_seqlens[b + 1] - start;
    if (len < 0 || len > max_seqlen) return ORACLE_ERR_ARG;
    for (int h = 0; h < heads; ++h) {
      for (int t = 0; t < nblk; ++t) {
        float* s_out = &scale[((size_t)h * batch + b) * nblk + t];
        int r0 = t * block;
        if (r0 >= len) {
          *s_out = 0.0f;
          continue;
        }
        int r1 = r0 + block < len ? r0 + block : len;
        float amax = 0.0f;
        for (int r = r0; r < r1; ++r) {
          const uint16_t* row = x + ((size_t)(start + r) * heads + h) * d;
          for (int c = 0; c < d; ++c) {
            float a = fabsf(half_bits_to_float(row[c]));
            if (a > amax) amax = a;
          }
        }
        float s = amax / 127.0f; /* one IEEE fp32 division */
        *s_out = s;
        for (int r = r0; r < r1; ++r) {
          const uint16_t* row = x + ((size_t)(start + r) * heads + h) * d;
          int8_t* qrow = x8 + ((size_t)(start + r) * heads + h) * d;
          for (int c = 0; c < d; ++c) {
            if (amax == 0.0f) {
              qrow[c] = 0;
              continue;
            }
            float ratio = half_bits_to_float(row[c]) / s; /* fp32 division */
            float rq = rintf(ratio); /* round half to even */
            if (rq > 127.0f) rq = 127.0f;
            if (rq < -127.0f) rq = -127.0f;
            qrow[c] = (int8_t)rq;
          }
        }
      }
    }
  }
  return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Routing words                                                            */
/* ------------------------------------------------------------------------ */

/* Last key tile that holds a legal (causal, in-sequence) key for query-tile
 * row m; -1 if the row holds no query of the sequence. */
static int last_legal_key_tile(int len, int m, int block_m, int block_n) {
  long first = (long)m * block_m;
  if (first >= len) return -1;
  long last_row = first + block_m - 1;
  if (last_row > len - 1) last_row = len - 1;
  return (int)(last_row / block_n); /* keys j <= last_row are legal */
}

/* route: uint8 [batch, hkv, tm_max, 64], nonzero = INT8.
 * mask: uint64 [batch, hkv, tm_max], tm_max = ceil(max_seqlen / block_m).
 * Bit j of a word is the route of key-tile group j; bits of groups that
 * hold no legal pair are 0. */
int oracle_pack_mask(const uint8_t* route, const int32_t* cu_seqlens,
                     int batch, int max_seqlen, int hkv, int block_m,
                     int block_n, int group, uint64_t* mask) {
  if (!route || !cu_seqlens || !mask || batch < 0 || hkv <= 0 ||
      block_m <= 0 || block_n <= 0 || group <= 0)
    return ORACLE_ERR_ARG;
  int tm = (max_seqlen + block_m - 1) / block_m;
  for (int b = 0; b < batch; ++b) {
    int len = cu_seqlens[b + 1] - cu_seqlens[b];
    if (len < 0 || len > max_seqlen) return ORACLE_ERR_ARG;
    for (int hk = 0; hk < hkv; ++hk) {
      for (int m = 0; m < tm; ++m) {
        size_t w = ((size_t)b * hkv + hk) * tm + m;
        int n_last = last_legal_key_tile(len, m, block_m, block_n);
        uint64_t word = 0;
        if (n_last >= 0) {
          int g_last = n_last / group;
          if (g_last >= 64) return ORACLE_ERR_GROUPS;
          for (int j = 0; j <= g_last; ++j)
            if (route[w * 64 + j]) word |= (uint64_t)1 << j;
        }
        mask[w] = word;
      }
    }
  }
  return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Attention                                                                */
/* ------------------------------------------------------------------------ */

typedef struct {
  int batch, max_seqlen, hq, hkv, d;
  const int32_t* cu_seqlens;
  const int32_t* head_map; /* [hq] -> KV head, NULL = contiguous groups */
  const uint16_t* q;       /* fp16 bits [T, hq, d] */
  const int8_t* q8;        /* [T, hq, d] */
  const float* q_scale;    /* [hq, batch, ceil(max_seqlen/quant_block_q)] */
  int kv_int8;             /* 0: k, v fp16; 1: k8, v8 + scales */
  const uint16_t* k;       /* fp16 bits [T, hkv, d] */
  const int8_t* k8;        /* [T, hkv, d] */
  const float* k_scale;    /* [hkv, batch, ceil(max_seqlen/quant_block_k)] */
  const uint16_t* v;       /* fp16 bits [T, hkv, d] */
  const int8_t* v8;        /* [T, hkv, d] */
  const float* v_scale;    /* [hkv, batch, ceil(max_seqlen/quant_block_k)] */
  const uint64_t* mask;    /* [batch, hkv, ceil(max_seqlen/block_m)] */
  int block_m, block_n, group;
  int fp16_only;           /* ignore the mask: every pair FP16 */
  int quant_block_q, quant_block_k;
  double softmax_scale;
  double* out;             /* [T, hq, d] */
  double* lse;             /* [hq, T] natural log, may be NULL */
  const int64_t* rows;     /* optional list of token indices; NULL = all */
  int64_t n_rows;
  int nthreads;            /* <= 0: all online cores */
  /* optional route statistics (whole problem, every head):
   * counts[0] = legal pairs routed FP16, counts[1] = legal pairs INT8 */
  int64_t* pair_counts;
} oracle_attn_args;

static int kv_head_of(const oracle_attn_args* a, int h) {
  if (a->head_map) return a->head_map[h];
  return h / (a->hq / a->hkv);
}

/* Route of the pair (i, j) of sequence b (local indices), KV head hk. */
static int route_bit(const oracle_attn_args* a, int b, int hk, int i, int j) {
  if (a->fp16_only) return 0;
  int tm = (a->max_seqlen + a->block_m - 1) / a->block_m;
  int m = i / a->block_m;
  int n = j / a->block_n;
  uint64_t word = a->mask[((size_t)b * a->hkv + hk) * tm + m];
  return (int)((word >> (n / a->group)) & 1u);
}

/* One query row: token index `tok` (global), head h.  Scratch holds
 * max_seqlen doubles. */
static void attend_row(const oracle_attn_args* a, int b, int h, int i,
                       double* s) {
  int start = a->cu_seqlens[b];
  int d = a->d;
  int hk = kv_head_of(a, h);
  int nbq = (a->max_seqlen + a->quant_block_q - 1) / a->quant_block_q;
  int nbk = (a->max_seqlen + a->quant_block_k - 1) / a->quant_block_k;
  size_t qoff = ((size_t)(start + i) * a->hq + h) * d;
  double sq = a->q8 ? (double)a->q_scale[((size_t)h * a->batch + b) * nbq +
                                          i / a->quant_block_q]
                    : 0.0;

  /* pass 1: materialise the legal scores s[0..i] (keys j <= i) */
  for (int j = 0; j <= i; ++j) {
    size_t koff = ((size_t)(start + j) * a->hkv + hk) * d;
    double sk = 0.0;
    if (a->k_scale)
      sk = (double)a->k_scale[((size_t)hk * a->batch + b) * nbk +
                              j / a->quant_block_k];
    if (route_bit(a, b, hk, i, j)) {
      int64_t acc = 0;
      for (int c = 0; c < d; ++c)
        acc += (int64_t)a->q8[qoff + c] * (int64_t)a->k8[koff + c];
      s[j] = a->softmax_scale * ((double)acc * sq * sk);
    } else if (a->kv_int8) {
      double acc = 0.0;
      for (int c = 0; c < d; ++c)
        acc += (double)half_bits_to_float(a->q[qoff + c]) *
               (double)a->k8[koff + c];
      s[j] = a->softmax_scale * (acc * sk);
    } else {
      double acc = 0.0;
      for (int c = 0; c < d; ++c)
        acc += (double)half_bits_to_float(a->q[qoff + c]) *
               (double)half_bits_to_float(a->k[koff + c]);
      s[j] = a->softmax_scale * acc;
    }
  }
  /* pass 2: softmax over the row, then the weighted sum of V */
  double mu = s[0];
  for (int j = 1; j <= i; ++j)
    if (s[j] > mu) mu = s[j];
  double l = 0.0;
  for (int j = 0; j <= i; ++j) {
    s[j] = exp(s[j] - mu);
    l += s[j];
  }
  double* o = a->out + qoff;
  for (int c = 0; c < d; ++c) o[c] = 0.0;
  for (int j = 0; j <= i; ++j) {
    size_t voff = ((size_t)(start + j) * a->hkv + hk) * d;
    double w = s[j] / l;
    if (a->kv_int8) {
      double sv = (double)a->v_scale[((size_t)hk * a->batch + b) * nbk +
                                     j / a->quant_block_k];
      for (int c = 0; c < d; ++c) o[c] += w * ((double)a->v8[voff + c] * sv);
    } else {
      for (int c = 0; c < d; ++c)
        o[c] += w * (double)half_bits_to_float(a->v[voff + c]);
    }
  }
  if (a->lse) {
    size_t total = (size_t)a->cu_seqlens[a->batch];
    a->lse[(size_t)h * total + start + i] = mu + log(l);
  }
}

typedef struct {
  const oracle_attn_args* a;
  int64_t next; /* shared work counter, guarded by lock */
  int64_t n_items;
  pthread_mutex_t lock;
  int failed;
} work_pool;

/* Work item = (token index, head) in token-major order. */
static int sequence_of(const oracle_attn_args* a, int64_t tok) {
  int lo = 0, hi = a->batch - 1;
  while (lo < hi) { /* last b with cu[b] <= tok */
    int mid = (lo + hi + 1) / 2;
    if (a->cu_seqlens[mid] <= tok) lo = mid; else hi = mid - 1;
  }
  return lo;
}

static void* worker(void* arg) {
  work_pool* pool = (work_pool*)arg;
  const oracle_attn_args* a = pool->a;
  double* s = (double*)malloc(sizeof(double) * (size_t)(a->max_seqlen + 1));
  if (!s) {
    pthread_mutex_lock(&pool->lock);
    pool->failed = 1;
    pthread_mutex_unlock(&pool->lock);
    return NULL;
  }
  const int64_t chunk = 16;
  for (;;) {
    pthread_mutex_lock(&pool->lock);
    int64_t first = pool->next;
    pool->next += chunk;
    pthread_mutex_unlock(&pool->lock);
    if (first >= pool->n_items) break;
    int64_t last = first + chunk < pool->n_items ? first + chunk : pool->n_items;
    for (int64_t it = first; it < last; ++it) {
      int64_t r = it / a->hq;
      int h = (int)(it % a->hq);
      int64_t tok = a->rows ? a->rows[r] : r;
      int b = sequence_of(a, tok);
      attend_row(a, b, h, (int)(tok - a->cu_seqlens[b]), s);
    }
  }
  free(s);
  return NULL;
}

int oracle_attn(const oracle_attn_args* a) {
  if (!a || !a->cu_seqlens || !a->q || !a->out || a->batch <= 0 ||
      a->hq <= 0 || a->hkv <= 0 || a->d <= 0 || a->block_m <= 0 ||
      a->block_n <= 0 || a->group <= 0 || a->quant_block_q <= 0 ||
      a->quant_block_k <= 0)
    return ORACLE_ERR_ARG;
  if (!a->head_map && a->hq % a->hkv != 0) return ORACLE_ERR_ARG;
  if (!a->fp16_only && (!a->mask || !a->q8 || !a->q_scale || !a->k8 ||
                        !a->k_scale))
    return ORACLE_ERR_ARG;
  if (a->kv_int8 && (!a->k8 || !a->k_scale || !a->v8 || !a->v_scale))
    return ORACLE_ERR_ARG;
  if (!a->kv_int8 && (!a->k || !a->v)) return ORACLE_ERR_ARG;
  for (int b = 0; b < a->batch; ++b) {
    int len = a->cu_seqlens[b + 1] - a->cu_seqlens[b];
    if (len < 0 || len > a->max_seqlen) return ORACLE_ERR_ARG;
  }
  int64_t total = a->cu_seqlens[a->batch];
  int64_t n_rows = a->rows ? a->n_rows : total;
  for (int64_t r = 0; a->rows && r < n_rows; ++r)
    if (a->rows[r] < 0 || a->rows[r] >= total) return ORACLE_ERR_ARG;

  if (a->pair_counts) {
    a->pair_counts[0] = a->pair_counts[1] = 0;
    for (int b = 0; b < a->batch; ++b) {
      int len = a->cu_seqlens[b + 1] - a->cu_seqlens[b];
      for (int h = 0; h < a->hq; ++h) {
        int hk = kv_head_of(a, h);
        for (int i = 0; i < len; ++i)
          for (int j = 0; j <= i; ++j)
            a->pair_counts[route_bit(a, b, hk, i, j)] += 1;
      }
    }
  }

  work_pool pool;
  pool.a = a;
  pool.next = 0;
  pool.n_items = n_rows * a->hq;
  pool.failed = 0;
  pthread_mutex_init(&pool.lock, NULL);
  int nt = a->nthreads > 0 ? a->nthreads : (int)sysconf(_SC_NPROCESSORS_ONLN);
  if (nt < 1) nt = 1;
  if (nt > 256) nt = 256;
  pthread_t th[256];
  int started = 0;
  for (int t = 0; t < nt; ++t)
    if (pthread_create(&th[t], NULL, worker, &pool) == 0) ++started;
  if (started == 0) worker(&pool);
  for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
  pthread_mutex_destroy(&pool.lock);
  return pool.failed ? ORACLE_ERR_ALLOC : ORACLE_OK;
}

/* INT32 score accumulators of every INT8-routed legal tile:
 * dump[b][h][m][n][r][c] = sum_k q8[m*BM + r][k] * k8[n*BN + c][k] for
 * rows m*BM + r < len and keys n*BN + c < len, including causally masked
 * positions inside the tile.  Other entries are left as they are. */
int oracle_qk_dump(const oracle_attn_args* a, int32_t* dump) {
  if (!a || !dump || !a->q8 || !a->k8 || !a->mask) return ORACLE_ERR_ARG;
  int tm = (a->max_seqlen + a->block_m - 1) / a->block_m;
  int tn = (a->max_seqlen + a->block_n - 1) / a->block_n;
  int bm = a->block_m, bn = a->block_n, d = a->d;
  for (int b = 0; b < a->batch; ++b) {
    int start = a->cu_seqlens[b];
    int len = a->cu_seqlens[b + 1] - start;
    for (int h = 0; h < a->hq; ++h) {
      int hk = kv_head_of(a, h);
      for (int m = 0; m < tm; ++m) {
        int n_last = last_legal_key_tile(len, m, bm, bn);
        uint64_t word = a->mask[((size_t)b * a->hkv + hk) * tm + m];
        for (int n = 0; n <= n_last; ++n) {
          if (!((word >> (n / a->group)) & 1u)) continue;
          for (int r = 0; r < bm && m * bm + r < len; ++r) {
            int i = m * bm + r;
            size_t qoff = ((size_t)(start + i) * a->hq + h) * d;
            for (int c = 0; c < bn && n * bn + c < len; ++c) {
              int j = n * bn + c;
              size_t koff = ((size_t)(start + j) * a->hkv + hk) * d;
              int64_t acc = 0;
              for (int k = 0; k < d; ++k)
                acc += (int64_t)a->q8[qoff + k] * (int64_t)a->k8[koff + k];
              size_t idx = ((((size_t)b * a->hq + h) * tm + m) * tn + n);
              dump[(idx * bm + r) * bn + c] = (int32_t)acc;
            }
          }
        }
      }
    }
  }
  return ORACLE_OK;
}
