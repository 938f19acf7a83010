/*
 * rpa_oracle.c -- plain, slow, fp64 CPU oracle for ragged paged attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library.
 *
 * What it computes (and where the pages state it):
 *   - "Ragged Paged Attention: A High-Performance and Flexible LLM Inference
 *     Kernel for TPU" (arXiv 2604.15464), abstract: one attention kernel over a
 *     ragged batch of paged sequences that mixes decode, prefill and mixed
 *     work, with the KV-cache update fused into the attention computation.
 *   - RPA talk summary (rocketrecap.com), 00:06:36: the newly projected K/V
 *     are written into the cache while the attention over the cache runs, so
 *     the attention sees the cache *after* the update.
 *   - same talk, glossary "FlashAttention": exact attention (no
 *     approximation), so the plain softmax(QK^T)V definition is the answer.
 *   - same talk, glossary "PagedAttention": a sequence's KV lives in
 *     non-contiguous fixed-size physical blocks; a per-sequence table maps
 *     logical block j to its physical page.
 *   - same talk, 00:11:09: the prefill numbers are quoted with and without a
 *     causal mask, so both variants exist.
 *
 * Readings where the pages are silent (each listed with its reason in the
 * design notes): causal masks are bottom-right aligned (new token i of a
 * sequence with c = kv_len - q_len context tokens sits at absolute position
 * c + i and sees keys 0..c+i); query head h reads KV head h / G with
 * G = Hq / Hkv; lse is the natural log of the sum of exp over the scaled,
 * visible scores.
 *
 * Layouts (row-major):  q [T, Hq, D]; k_new, v_new [T, Hkv, D];
 * caches [num_pages, P, Hkv, D]; page_table [S, max_pages] int32;
 * cu_q_lens [S+1]; kv_lens [S]; out [T, Hq, D] fp64; lse [T, Hq] fp64.
 * dtype 0 = fp32, 1 = bf16 (bit pattern, widened exactly to fp64).
 *
 * Every step is written in the order the definition states it: scatter
 * first, then for each (sequence, query head, query row) gather the logical
 * K/V, score, mask, softmax, weight V.  No blocking, fusion or reordering.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG -1
#define ORACLE_ERR_LENGTHS -2
#define ORACLE_ERR_PAGE -3

/* Exact widening of one stored element to fp64. */
static double elem(const void *base, size_t idx, int dtype) {
  if (dtype == 0) return (double)((const float *)base)[idx];
  uint32_t bits = (uint32_t)((const uint16_t *)base)[idx] << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

static size_t elem_size(int dtype) { return dtype == 0 ? 4u : 2u; }

typedef struct {
  const int32_t *page_table;
  int32_t max_pages;
  const int32_t *cu_q_lens;
  const int32_t *kv_lens;
  int32_t num_seqs, hq, hkv, d, p, num_pages, dtype;
} geom;

/* Checks every length and every page-table entry a sequence will touch. */
static int check(const geom *g) {
  if (g->num_seqs < 0 || g->hq <= 0 || g->hkv <= 0 || g->d <= 0 || g->p <= 0 ||
      g->hq % g->hkv != 0 || (g->dtype != 0 && g->dtype != 1))
    return ORACLE_ERR_ARG;
  if (g->num_seqs > 0 && g->cu_q_lens[0] != 0) return ORACLE_ERR_LENGTHS;
  for (int s = 0; s < g->num_seqs; ++s) {
    int32_t ql = g->cu_q_lens[s + 1] - g->cu_q_lens[s];
    int32_t kv = g->kv_lens[s];
    if (ql < 0 || kv < ql) return ORACLE_ERR_LENGTHS;
    int32_t npages = (kv + g->p - 1) / g->p;
    if (npages > g->max_pages) return ORACLE_ERR_LENGTHS;
    for (int32_t j = 0; j < npages; ++j) {
      int32_t pg = g->page_table[(size_t)s * g->max_pages + j];
      if (pg < 0 || pg >= g->num_pages) return ORACLE_ERR_PAGE;
    }
  }
  return ORACLE_OK;
}

/* Flat index of element (logical position pos, kv head h, dim 0) of sequence
 * s inside a paged cache: physical page = page_table[s][pos / P], slot =
 * pos % P (PagedAttention glossary entry of the talk summary). */
static size_t cache_index(const geom *g, int s, int32_t pos, int h) {
  int32_t page = g->page_table[(size_t)s * g->max_pages + pos / g->p];
  int32_t slot = pos % g->p;
  return (((size_t)page * g->p + slot) * g->hkv + h) * (size_t)g->d;
}

/* Step 1, the fused cache update (talk summary 00:06:36): for each sequence
 * with c = kv_len - q_len, new token i is stored, bit for bit, at logical
 * position c + i of its page chain. */
int rpa_oracle_scatter(const void *k_new, const void *v_new, void *k_cache,
                       void *v_cache, const int32_t *page_table,
                       int32_t max_pages, const int32_t *cu_q_lens,
                       const int32_t *kv_lens, int32_t num_seqs, int32_t hq,
                       int32_t hkv, int32_t d, int32_t p, int32_t num_pages,
                       int32_t dtype) {
  geom g = {page_table, max_pages, cu_q_lens, kv_lens, num_seqs,
            hq,         hkv,       d,         p,       num_pages, dtype};
  int rc = check(&g);
  if (rc) return rc;
  size_t es = elem_size(dtype);
  size_t row_bytes = (size_t)hkv * d * es; /* all kv heads of one token */
  for (int s = 0; s < num_seqs; ++s) {
    int32_t ql = cu_q_lens[s + 1] - cu_q_lens[s];
    int32_t c = kv_lens[s] - ql;
    for (int32_t i = 0; i < ql; ++i) {
      size_t src = (size_t)(cu_q_lens[s] + i) * hkv * d * es;
      size_t dst = cache_index(&g, s, c + i, 0) * es;
      memcpy((char *)k_cache + dst, (const char *)k_new + src, row_bytes);
      memcpy((char *)v_cache + dst, (const char *)v_new + src, row_bytes);
    }
  }
  return ORACLE_OK;
}

/* Step 2, attention of one query row (sequence s, new token i, query head h)
 * over the updated cache.  Writes out_row[D] and *lse_row; if weights is not
 * NULL it also receives the normalised softmax weights over all kv_len keys
 * (0 for masked keys). */
static void attend_row(const geom *g, const void *q, const void *k_cache,
                       const void *v_cache, double scale, int causal, int s,
                       int32_t i, int h, double *scores, double *out_row,
                       double *lse_row, double *weights) {
  int32_t ql = g->cu_q_lens[s + 1] - g->cu_q_lens[s];
  int32_t kv = g->kv_lens[s];
  int32_t c = kv - ql;
  int hk = h / (g->hq / g->hkv); /* GQA: contiguous groups of G query heads */
  size_t qoff = ((size_t)(g->cu_q_lens[s] + i) * g->hq + h) * (size_t)g->d;

  /* scores over the visible keys: j < kv_len and, if causal, j <= c + i */
  int32_t nvis = causal ? c + i + 1 : kv;
  double m = -INFINITY;
  for (int32_t j = 0; j < nvis; ++j) {
    size_t koff = cache_index(g, s, j, hk);
    double dot = 0.0;
    for (int t = 0; t < g->d; ++t)
      dot += elem(q, qoff + t, g->dtype) * elem(k_cache, koff + t, g->dtype);
    scores[j] = scale * dot;
    if (scores[j] > m) m = scores[j];
  }
  /* softmax: l = sum exp(S - m); out = sum exp(S - m) V / l; lse = m + ln l */
  double l = 0.0;
  for (int32_t j = 0; j < nvis; ++j) l += exp(scores[j] - m);
  for (int t = 0; t < g->d; ++t) out_row[t] = 0.0;
  for (int32_t j = 0; j < nvis; ++j) {
    double w = exp(scores[j] - m) / l;
    size_t voff = cache_index(g, s, j, hk);
    for (int t = 0; t < g->d; ++t)
      out_row[t] += w * elem(v_cache, voff + t, g->dtype);
    if (weights) weights[j] = w;
  }
  if (weights)
    for (int32_t j = nvis; j < kv; ++j) weights[j] = 0.0;
  *lse_row = m + log(l);
}

/* The whole forward pass: scatter, then every query row of every sequence.
 * k_cache / v_cache are host copies that this call updates in place. */
int rpa_oracle_forward(const void *q, const void *k_new, const void *v_new,
                       void *k_cache, void *v_cache, const int32_t *page_table,
                       int32_t max_pages, const int32_t *cu_q_lens,
                       const int32_t *kv_lens, int32_t num_seqs, int32_t hq,
                       int32_t hkv, int32_t d, int32_t p, int32_t num_pages,
                       int32_t dtype, double scale, int32_t causal, double *out,
                       double *lse, int32_t num_threads) {
  geom g = {page_table, max_pages, cu_q_lens, kv_lens, num_seqs,
            hq,         hkv,       d,         p,       num_pages, dtype};
  int rc = rpa_oracle_scatter(k_new, v_new, k_cache, v_cache, page_table,
                              max_pages, cu_q_lens, kv_lens, num_seqs, hq, hkv,
                              d, p, num_pages, dtype);
  if (rc) return rc;
  int32_t max_kv = 1;
  for (int s = 0; s < num_seqs; ++s)
    if (kv_lens[s] > max_kv) max_kv = kv_lens[s];
  long npairs = (long)num_seqs * hq;
#ifdef _OPENMP
  if (num_threads > 0) omp_set_num_threads(num_threads);
#else
  (void)num_threads;
#endif
#pragma omp parallel
  {
    double *scores = (double *)malloc(sizeof(double) * (size_t)max_kv);
#pragma omp for schedule(dynamic, 1)
    for (long pair = 0; pair < npairs; ++pair) {
      int s = (int)(pair / hq), h = (int)(pair % hq);
      int32_t ql = cu_q_lens[s + 1] - cu_q_lens[s];
      for (int32_t i = 0; i < ql; ++i) {
        size_t row = (size_t)(cu_q_lens[s] + i) * hq + h;
        attend_row(&g, q, k_cache, v_cache, scale, causal, s, i, h, scores,
                   out + row * d, lse + row, NULL);
      }
    }
    free(scores);
  }
  return ORACLE_OK;
}

/* Attention of an explicit list of query rows over an ALREADY UPDATED cache
 * (call rpa_oracle_scatter first).  rows[n] are global token indices in
 * [0, T); heads[n] their query heads.  out_rows [n, D], lse_rows [n]. */
int rpa_oracle_attend_rows(const void *q, const void *k_cache,
                           const void *v_cache, const int32_t *page_table,
                           int32_t max_pages, const int32_t *cu_q_lens,
                           const int32_t *kv_lens, int32_t num_seqs, int32_t hq,
                           int32_t hkv, int32_t d, int32_t p, int32_t num_pages,
                           int32_t dtype, double scale, int32_t causal,
                           int32_t n, const int32_t *rows, const int32_t *heads,
                           double *out_rows, double *lse_rows,
                           int32_t num_threads) {
  geom g = {page_table, max_pages, cu_q_lens, kv_lens, num_seqs,
            hq,         hkv,       d,         p,       num_pages, dtype};
  int rc = check(&g);
  if (rc) return rc;
  int32_t total = num_seqs > 0 ? cu_q_lens[num_seqs] : 0;
  for (int32_t r = 0; r < n; ++r)
    if (rows[r] < 0 || rows[r] >= total || heads[r] < 0 || heads[r] >= hq)
      return ORACLE_ERR_ARG;
  int32_t max_kv = 1;
  for (int s = 0; s < num_seqs; ++s)
    if (kv_lens[s] > max_kv) max_kv = kv_lens[s];
#ifdef _OPENMP
  if (num_threads > 0) omp_set_num_threads(num_threads);
#else
  (void)num_threads;
#endif
#pragma omp parallel
  {
    double *scores = (double *)malloc(sizeof(double) * (size_t)max_kv);
#pragma omp for schedule(dynamic, 1)
    for (int32_t r = 0; r < n; ++r) {
      /* the sequence that owns global token rows[r] */
      int s = 0;
      while (cu_q_lens[s + 1] <= rows[r]) ++s;
      attend_row(&g, q, k_cache, v_cache, scale, causal, s,
                 rows[r] - cu_q_lens[s], heads[r], scores,
                 out_rows + (size_t)r * d, lse_rows + r, NULL);
    }
    free(scores);
  }
  return ORACLE_OK;
}

/* Softmax weights of one query row over its kv_len keys (masked keys get 0),
 * over an already updated cache.  Exposed so tests can check that every row
 * of weights sums to one. */
int rpa_oracle_row_weights(const void *q, const void *k_cache,
                           const void *v_cache, const int32_t *page_table,
                           int32_t max_pages, const int32_t *cu_q_lens,
                           const int32_t *kv_lens, int32_t num_seqs, int32_t hq,
                           int32_t hkv, int32_t d, int32_t p, int32_t num_pages,
                           int32_t dtype, double scale, int32_t causal,
                           int32_t seq, int32_t i, int32_t h, double *weights) {
  geom g = {page_table, max_pages, cu_q_lens, kv_lens, num_seqs,
            hq,         hkv,       d,         p,       num_pages, dtype};
  int rc = check(&g);
  if (rc) return rc;
  if (seq < 0 || seq >= num_seqs || h < 0 || h >= hq || i < 0 ||
      i >= cu_q_lens[seq + 1] - cu_q_lens[seq])
    return ORACLE_ERR_ARG;
  double *scores = (double *)malloc(sizeof(double) * (size_t)(kv_lens[seq] + 1));
  double *orow = (double *)malloc(sizeof(double) * (size_t)d);
  double l;
  attend_row(&g, q, k_cache, v_cache, scale, causal, seq, i, h, scores, orow,
             &l, weights);
  free(scores);
  free(orow);
  return ORACLE_OK;
}

int rpa_oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
