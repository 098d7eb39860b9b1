/*
 * attn_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct CPU statement of exact softmax attention
 * in double precision.  It exists so that tests, the smoke check and the
 * benchmark's CPU-baseline leg can check the CUDA path against it.  Nothing
 * in the product path may link, load or call this file, and it shares no
 * code, header or constant with the CUDA library.
 *
 * What it follows (page titles and sections of the source notes):
 *   - "Attention Kernel", section "问题与成本" (problem and cost):
 *       P = softmax(Q K^T / sqrt(d_h) + M),  O = P V,
 *       Q in R^{B x A x S_q x d_h},  K, V in R^{B x A_kv x S_k x d_h}.
 *     Several query heads share one KV head (GQA); the head mapping is the
 *     contiguous one, kv = hq / (Hq / Hkv).
 *   - "Attention Kernel", section "Online softmax": the (m, l, o) state, the
 *     merge rule m' = max(m, m_b), l' = e^{m-m'} l + e^{m_b-m'} l_b,
 *     o' = e^{m-m'} o + e^{m_b-m'} o_b, and O = o / l; a row whose scores are
 *     all -inf returns the agreed zero output rather than NaN.
 *   - "Attention Kernel", section "Blockwise reference": the blockwise walk
 *     over one score row that skips blocks with no finite score and returns
 *     zeros when the normaliser is zero; mismatched score/value rows are
 *     rejected.
 *   - "Attention Kernel", section "Paged 与 ragged KV": logical token t lives
 *     in block floor(t / q) at offset t mod q, and the block table gives the
 *     physical page.
 *   - "Attention 算子加速史" (FlashAttention history), FAQ Q3: subtract the row
 *     maximum before exponentiating.
 *
 * Readings where the notes are silent (each also listed in the design notes):
 *   - LSE is the natural log of sum_j exp(scale * q.k_j) over visible keys;
 *     a row with no visible key has O = 0 and LSE = -inf.
 *   - The scale multiplies the dot product; the mask (0 or -inf) is added
 *     after scaling.
 *   - Causal alignment is bottom-right: with k_len keys visible to sequence
 *     b, key j is visible to query row i iff j < k_len and, when causal,
 *     j <= i + (k_len - Sq).
 *   - Programmable masks ("Attention Kernel", section "可编程 mask"), both
 *     with causal: a sliding window w > 0 keeps only the w keys ending at the
 *     row's position p = i + (k_len - Sq), i.e. j > p - w; a prefix P > 0
 *     makes keys j < P visible to every row (prefix-LM).  Not both at once.
 *     A block mask (uint8 [B, mask_heads, ceil(Sq/128), ceil(Sk/128)],
 *     mask_heads 1 or Hq) hides every key j of query row i whose block
 *     entry [b][h][i/128][j/128] is 0 (block-sparse attention).
 *
 * Inputs to the attention routines are bf16 bit patterns (uint16); this
 * file widens them to double itself (a bf16 value is the top half of an
 * IEEE binary32, so the widening is exact).  All arithmetic is in double.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_TABLE 2

static double bf16_to_double(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* ------------------------------------------------------------------------ */
/* One score row against its value rows: the plain definition.              */
/* ------------------------------------------------------------------------ */

/*
 * softmax(s) @ v for one row, written out directly: m = max_j s_j; if every
 * s_j is -inf the row is empty (O = 0, LSE = -inf); otherwise
 * p_j = exp(s_j - m), l = sum p_j, O = sum_j p_j v_j / l, LSE = m + ln l.
 * n_scores must equal n_value_rows (the notes' blockwise reference rejects a
 * mismatch; so does this).
 */
int oracle_softmax_attend(const double* s, int n_scores, const double* v,
                          int n_value_rows, int dv, double* o, double* lse) {
  if (n_scores != n_value_rows || n_scores < 0 || dv <= 0 || !o || !lse ||
      (n_scores > 0 && (!s || !v)))
    return ORACLE_ERR_ARG;
  double m = -INFINITY;
  for (int j = 0; j < n_scores; ++j)
    if (s[j] > m) m = s[j];
  for (int t = 0; t < dv; ++t) o[t] = 0.0;
  if (m == -INFINITY) {
    *lse = -INFINITY;
    return ORACLE_OK;
  }
  double l = 0.0;
  for (int j = 0; j < n_scores; ++j) {
    if (s[j] == -INFINITY) continue;
    double p = exp(s[j] - m);
    l += p;
    for (int t = 0; t < dv; ++t) o[t] += p * v[(size_t)j * dv + t];
  }
  for (int t = 0; t < dv; ++t) o[t] /= l;
  *lse = m + log(l);
  return ORACLE_OK;
}

/*
 * The same row computed block by block with the online (m, l, o) state, in
 * the block order given (block_order[i] = index of the i-th block to visit;
 * NULL means ascending).  Blocks whose scores are all -inf are skipped, and
 * a zero normaliser at the end yields the zero row, as the notes' blockwise
 * reference does.  Used only to check that block size and order do not
 * change the result.
 */
int oracle_online_attend(const double* s, int n_scores, const double* v,
                         int n_value_rows, int dv, int block_size,
                         const int* block_order, double* o, double* lse) {
  if (n_scores != n_value_rows || n_scores < 0 || dv <= 0 || block_size <= 0 ||
      !o || !lse || (n_scores > 0 && (!s || !v)))
    return ORACLE_ERR_ARG;
  int n_blocks = (n_scores + block_size - 1) / block_size;
  double* num = (double*)calloc((size_t)dv, sizeof(double));
  double* blk = (double*)calloc((size_t)dv, sizeof(double));
  if (!num || !blk) {
    free(num);
    free(blk);
    return ORACLE_ERR_ARG;
  }
  if (block_order) { /* must be a permutation of 0..n_blocks-1 */
    char* seen = (char*)calloc((size_t)n_blocks + 1, 1);
    int ok = seen != NULL;
    for (int i = 0; ok && i < n_blocks; ++i) {
      int b = block_order[i];
      if (b < 0 || b >= n_blocks || seen[b]) ok = 0;
      else seen[b] = 1;
    }
    free(seen);
    if (!ok) {
      free(num);
      free(blk);
      return ORACLE_ERR_ARG;
    }
  }
  double m = -INFINITY, l = 0.0;
  for (int i = 0; i < n_blocks; ++i) {
    int b = block_order ? block_order[i] : i;
    int j0 = b * block_size;
    int j1 = j0 + block_size < n_scores ? j0 + block_size : n_scores;
    double mb = -INFINITY;
    for (int j = j0; j < j1; ++j)
      if (s[j] > mb) mb = s[j];
    if (mb == -INFINITY) continue; /* nothing finite in this block */
    /* local state of the block: l_b = sum e^{s-m_b}, o_b = sum e^{s-m_b} v */
    double lb = 0.0;
    for (int t = 0; t < dv; ++t) blk[t] = 0.0;
    for (int j = j0; j < j1; ++j) {
      if (s[j] == -INFINITY) continue;
      double w = exp(s[j] - mb);
      lb += w;
      for (int t = 0; t < dv; ++t) blk[t] += w * v[(size_t)j * dv + t];
    }
    /* merge rule */
    double mn = m > mb ? m : mb;
    double a_old = (m == -INFINITY) ? 0.0 : exp(m - mn);
    double a_blk = exp(mb - mn);
    l = a_old * l + a_blk * lb;
    for (int t = 0; t < dv; ++t) num[t] = a_old * num[t] + a_blk * blk[t];
    m = mn;
  }
  if (l > 0.0) {
    for (int t = 0; t < dv; ++t) o[t] = num[t] / l;
    *lse = m + log(l);
  } else {
    for (int t = 0; t < dv; ++t) o[t] = 0.0;
    *lse = -INFINITY;
  }
  free(num);
  free(blk);
  return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Prefill: Q [B,Hq,Sq,d], K,V [B,Hkv,Sk,d], all contiguous, bf16 bits.     */
/* ------------------------------------------------------------------------ */

typedef struct {
  const uint16_t *q, *k, *v;
  int B, Hq, Hkv, Sq, Sk, d, causal, window, prefix, mask_heads;
  const uint8_t* block_mask;
  double scale;
  const int32_t* k_lens;
  const int64_t* rows; /* flat row ids (b*Hq + hq)*Sq + i, or NULL = all */
  int64_t n_rows;
  double *o, *lse;
  int64_t begin, end; /* this worker's slice of rows */
  int status;
} prefill_job;

/* Per-worker copy of one (sequence, KV head)'s keys and values in double. */
typedef struct {
  int b, kvh;
  double *k, *v, *qrow, *s;
} prefill_scratch;

static int prefill_row(const prefill_job* J, int64_t r, prefill_scratch* W) {
  int64_t flat = J->rows ? J->rows[r] : r;
  int64_t per_b = (int64_t)J->Hq * J->Sq;
  if (flat < 0 || flat >= (int64_t)J->B * per_b) return ORACLE_ERR_ARG;
  int b = (int)(flat / per_b);
  int hq = (int)((flat / J->Sq) % J->Hq);
  int i = (int)(flat % J->Sq);
  int g = J->Hq / J->Hkv;
  int kvh = hq / g; /* contiguous GQA groups */
  int d = J->d;
  int klen = J->k_lens ? J->k_lens[b] : J->Sk;
  if (klen < 0 || klen > J->Sk) return ORACLE_ERR_ARG;
  if (W->b != b || W->kvh != kvh) {
    const uint16_t* kp = J->k + ((size_t)b * J->Hkv + kvh) * (size_t)J->Sk * d;
    const uint16_t* vp = J->v + ((size_t)b * J->Hkv + kvh) * (size_t)J->Sk * d;
    for (size_t e = 0; e < (size_t)J->Sk * d; ++e) {
      W->k[e] = bf16_to_double(kp[e]);
      W->v[e] = bf16_to_double(vp[e]);
    }
    W->b = b;
    W->kvh = kvh;
  }
  const uint16_t* qp = J->q + (((size_t)b * J->Hq + hq) * J->Sq + i) * d;
  for (int t = 0; t < d; ++t) W->qrow[t] = bf16_to_double(qp[t]);
  int64_t pos = (int64_t)i + ((int64_t)klen - J->Sq); /* bottom-right causal alignment */
  for (int j = 0; j < J->Sk; ++j) {
    int visible = j < klen;
    if (J->causal) {
      visible = visible && ((int64_t)j <= pos || (int64_t)j < J->prefix);
      if (J->window > 0) visible = visible && (int64_t)j > pos - J->window;
    }
    if (J->block_mask) {
      int64_t n_qt = (J->Sq + 127) / 128, n_kt = (J->Sk + 127) / 128;
      int64_t h = J->mask_heads == 1 ? 0 : hq;
      visible = visible &&
                J->block_mask[(((int64_t)b * J->mask_heads + h) * n_qt + i / 128) * n_kt + j / 128];
    }
    if (!visible) {
      W->s[j] = -INFINITY;
      continue;
    }
    double dot = 0.0;
    for (int t = 0; t < d; ++t) dot += W->qrow[t] * W->k[(size_t)j * d + t];
    W->s[j] = J->scale * dot; /* scale, then the additive 0 / -inf mask */
  }
  return oracle_softmax_attend(W->s, J->Sk, W->v, J->Sk, d, J->o + (size_t)r * d, J->lse + r);
}

static void* prefill_worker(void* arg) {
  prefill_job* J = (prefill_job*)arg;
  size_t sk = J->Sk > 0 ? (size_t)J->Sk : 1;
  prefill_scratch W;
  W.b = -1;
  W.kvh = -1;
  W.k = (double*)malloc(sk * (size_t)J->d * sizeof(double));
  W.v = (double*)malloc(sk * (size_t)J->d * sizeof(double));
  W.qrow = (double*)malloc((size_t)J->d * sizeof(double));
  W.s = (double*)malloc(sk * sizeof(double));
  J->status = (W.k && W.v && W.qrow && W.s) ? ORACLE_OK : ORACLE_ERR_ARG;
  for (int64_t r = J->begin; J->status == ORACLE_OK && r < J->end; ++r)
    J->status = prefill_row(J, r, &W);
  free(W.k);
  free(W.v);
  free(W.qrow);
  free(W.s);
  return NULL;
}

/*
 * Exact attention for the listed query rows (rows == NULL: every row, in
 * [B,Hq,Sq] order).  o is [n_rows, d], lse is [n_rows].  k_lens (nullable)
 * gives the number of leading keys visible per sequence.  Work is split over
 * n_threads POSIX threads by rows; each row is computed independently.
 */
int oracle_attn_fwd_rows_blocks(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                int B, int Hq, int Hkv, int Sq, int Sk, int d, int causal,
                                double scale, const int32_t* k_lens, int window, int prefix,
                                const uint8_t* block_mask, int mask_heads, const int64_t* rows,
                                int64_t n_rows, double* o, double* lse, int n_threads) {
  if (!q || (Sk > 0 && (!k || !v)) || !o || !lse || B < 1 || Hq < 1 || Hkv < 1 ||
      Sq < 1 || Sk < 0 || d < 1 || Hq % Hkv != 0 || n_rows < 0 || !isfinite(scale))
    return ORACLE_ERR_ARG;
  if (window < 0 || prefix < 0 || (window > 0 && prefix > 0) ||
      ((window > 0 || prefix > 0) && !causal))
    return ORACLE_ERR_ARG;
  if (block_mask && mask_heads != 1 && mask_heads != Hq) return ORACLE_ERR_ARG;
  if (!rows && n_rows != (int64_t)B * Hq * Sq) return ORACLE_ERR_ARG;
  if (n_threads < 1) n_threads = 1;
  if ((int64_t)n_threads > n_rows) n_threads = n_rows > 0 ? (int)n_rows : 1;
  prefill_job* jobs = (prefill_job*)calloc((size_t)n_threads, sizeof(prefill_job));
  pthread_t* th = (pthread_t*)calloc((size_t)n_threads, sizeof(pthread_t));
  if (!jobs || !th) {
    free(jobs);
    free(th);
    return ORACLE_ERR_ARG;
  }
  for (int w = 0; w < n_threads; ++w) {
    prefill_job* J = &jobs[w];
    J->q = q; J->k = k; J->v = v;
    J->B = B; J->Hq = Hq; J->Hkv = Hkv; J->Sq = Sq; J->Sk = Sk; J->d = d;
    J->causal = causal; J->scale = scale; J->k_lens = k_lens;
    J->window = window; J->prefix = prefix;
    J->block_mask = block_mask; J->mask_heads = mask_heads;
    J->rows = rows; J->n_rows = n_rows; J->o = o; J->lse = lse;
    J->begin = n_rows * w / n_threads;
    J->end = n_rows * (w + 1) / n_threads;
  }
  for (int w = 1; w < n_threads; ++w) pthread_create(&th[w], NULL, prefill_worker, &jobs[w]);
  prefill_worker(&jobs[0]);
  int status = ORACLE_OK;
  for (int w = 0; w < n_threads; ++w) {
    if (w > 0) pthread_join(th[w], NULL);
    if (jobs[w].status != ORACLE_OK) status = jobs[w].status;
  }
  free(jobs);
  free(th);
  return status;
}

/* oracle_attn_fwd_rows_blocks without a block mask. */
int oracle_attn_fwd_rows_masked(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                int B, int Hq, int Hkv, int Sq, int Sk, int d, int causal,
                                double scale, const int32_t* k_lens, int window, int prefix,
                                const int64_t* rows, int64_t n_rows, double* o, double* lse,
                                int n_threads) {
  return oracle_attn_fwd_rows_blocks(q, k, v, B, Hq, Hkv, Sq, Sk, d, causal, scale, k_lens,
                                     window, prefix, NULL, 1, rows, n_rows, o, lse, n_threads);
}

/* oracle_attn_fwd_rows_masked without a window or prefix. */
int oracle_attn_fwd_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         int B, int Hq, int Hkv, int Sq, int Sk, int d, int causal,
                         double scale, const int32_t* k_lens, const int64_t* rows,
                         int64_t n_rows, double* o, double* lse, int n_threads) {
  return oracle_attn_fwd_rows_masked(q, k, v, B, Hq, Hkv, Sq, Sk, d, causal, scale, k_lens, 0, 0,
                                     rows, n_rows, o, lse, n_threads);
}

/* ------------------------------------------------------------------------ */
/* Decode over a paged KV cache: q [B,Hq,d]; caches [num_pages,page,Hkv,d]. */
/* ------------------------------------------------------------------------ */

typedef struct {
  const uint16_t *q, *kc, *vc;
  const int32_t *table, *seq_lens;
  int B, Hq, Hkv, d, page_size, max_pages, num_pages;
  double scale;
  double *o, *lse;
  int begin, end; /* slice of (b, hq) pairs */
  int status;
} decode_job;

static void* decode_worker(void* arg) {
  decode_job* J = (decode_job*)arg;
  int d = J->d, g = J->Hq / J->Hkv;
  size_t cap = (size_t)J->max_pages * J->page_size;
  if (cap == 0) cap = 1;
  double* s = (double*)malloc(cap * sizeof(double));
  double* vrows = (double*)malloc(cap * (size_t)d * sizeof(double));
  J->status = (s && vrows) ? ORACLE_OK : ORACLE_ERR_ARG;
  for (int p = J->begin; J->status == ORACLE_OK && p < J->end; ++p) {
    int b = p / J->Hq, hq = p % J->Hq, kvh = hq / g;
    int len = J->seq_lens[b];
    if (len < 0 || (int64_t)len > (int64_t)J->max_pages * J->page_size) {
      J->status = ORACLE_ERR_TABLE;
      break;
    }
    const uint16_t* qp = J->q + ((size_t)b * J->Hq + hq) * d;
    for (int t = 0; t < len; ++t) {
      /* logical token t -> block t / page_size, offset t mod page_size */
      int blk = t / J->page_size, off = t % J->page_size;
      int page = J->table[(size_t)b * J->max_pages + blk];
      if (page < 0 || page >= J->num_pages) {
        J->status = ORACLE_ERR_TABLE;
        break;
      }
      size_t base = (((size_t)page * J->page_size + off) * J->Hkv + kvh) * d;
      double dot = 0.0;
      for (int c = 0; c < d; ++c) dot += bf16_to_double(qp[c]) * bf16_to_double(J->kc[base + c]);
      s[t] = J->scale * dot;
      for (int c = 0; c < d; ++c) vrows[(size_t)t * d + c] = bf16_to_double(J->vc[base + c]);
    }
    if (J->status != ORACLE_OK) break;
    J->status = oracle_softmax_attend(s, len, vrows, len, d, J->o + (size_t)p * d, J->lse + p);
  }
  free(s);
  free(vrows);
  return NULL;
}

/*
 * Exact single-query attention of every (sequence, query head) against the
 * sequence's first seq_lens[b] tokens, gathered through the block table.
 * o is [B, Hq, d], lse is [B, Hq].  Returns ORACLE_ERR_TABLE for a page id
 * outside [0, num_pages) or a length beyond max_pages * page_size.
 */
int oracle_decode_paged(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                        const int32_t* block_table, const int32_t* seq_lens, int B, int Hq,
                        int Hkv, int d, int page_size, int max_pages, int num_pages,
                        double scale, double* o, double* lse, int n_threads) {
  if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !o || !lse || B < 1 ||
      Hq < 1 || Hkv < 1 || d < 1 || Hq % Hkv != 0 || page_size < 1 || max_pages < 0 ||
      num_pages < 0 || !isfinite(scale))
    return ORACLE_ERR_ARG;
  int n = B * Hq;
  if (n_threads < 1) n_threads = 1;
  if (n_threads > n) n_threads = n;
  decode_job* jobs = (decode_job*)calloc((size_t)n_threads, sizeof(decode_job));
  pthread_t* th = (pthread_t*)calloc((size_t)n_threads, sizeof(pthread_t));
  if (!jobs || !th) {
    free(jobs);
    free(th);
    return ORACLE_ERR_ARG;
  }
  for (int w = 0; w < n_threads; ++w) {
    decode_job* J = &jobs[w];
    J->q = q; J->kc = k_cache; J->vc = v_cache; J->table = block_table;
    J->seq_lens = seq_lens; J->B = B; J->Hq = Hq; J->Hkv = Hkv; J->d = d;
    J->page_size = page_size; J->max_pages = max_pages; J->num_pages = num_pages;
    J->scale = scale; J->o = o; J->lse = lse;
    J->begin = (int)((int64_t)n * w / n_threads);
    J->end = (int)((int64_t)n * (w + 1) / n_threads);
  }
  for (int w = 1; w < n_threads; ++w) pthread_create(&th[w], NULL, decode_worker, &jobs[w]);
  decode_worker(&jobs[0]);
  int status = ORACLE_OK;
  for (int w = 0; w < n_threads; ++w) {
    if (w > 0) pthread_join(th[w], NULL);
    if (jobs[w].status != ORACLE_OK) status = jobs[w].status;
  }
  free(jobs);
  free(th);
  return status;
}
