/*
 * oracle.c -- plain, slow, fp64 CPU oracle for the DeepSeek Sparse Attention
 * (DSA) hot path: lightning-indexer scores -> per-query top-k -> sparse
 * attention in the MQA mode of MLA.
 *
 * THIS IS TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load it.  It shares no code, header, table or
 * constant with the CUDA library, and the CUDA library never calls it.
 *
 * Everything is computed in double precision straight from the definitions,
 * one query row at a time, with no blocking, fusion or reordering.  OpenMP
 * only spreads independent work over host cores: query rows, or the scores
 * of one row (oracle_indexer_at).
 *
 * Sources (the pages this follows):
 *  - "DeepSeek V3.2 and the lightning indexer" (montana-research blog),
 *    section "How the lightning indexer works": a handful of FP8 indexer heads
 *    each take a ReLU-clipped dot product of the query with an earlier token,
 *    and a per-head weight combines them into one score; a query keeps its
 *    2,048 highest-scoring entries and its attention reads nothing else; under
 *    MLA's MQA form every query head shares the selected latents, so there is
 *    one selection per query position.
 *  - "DeepSeek-V3.2" (atlas.lewiswon.me), "Design overview" and the
 *    "Inference efficiency" row of the spec sheet: a few indexer heads score
 *    every query against all earlier tokens with ReLU and per-head weights;
 *    token-level top-k with k = 2048 per query; the main attention reads only
 *    the chosen latents.
 *  - "DeepSeek-V3.2 ... (introducing DSA)" (phantomic12 paper record): each
 *    (query, KV) pair gets a single scalar from the FP8 ReLU indexer, and the
 *    attention reads the k best per query.
 *
 * Readings where the pages are silent:
 *  - causal: the query at absolute position p may use keys 0..p (self
 *    included); in a sequence with n_k keys and n_q queries the local query i
 *    sits at p = (n_k - n_q) + i;
 *  - indexer: I[t,s] = sum_j w[t,j] * max(0, qhat[t,j,:] . khat[s,:]) with
 *    qhat = e4m3(q8) * q_scale[t,j] and khat = e4m3(k8) * k_scale[s];
 *  - top-k: the min(k, p+1) largest scores, ties to the lower index, -0 equal
 *    to +0, emitted in ascending index order and padded with -1;
 *  - attention: o[t,h] = sum_s softmax_s(scale * q[t,h,:] . c[s,:]) * c[s,0:d_v]
 *    over the selected set, lse = log sum_s exp(scale * q . c);
 *  - indexer training signal (oracle_indexer_kl_at): target p = the head
 *    average of the attention distributions over the selected set, loss
 *    KL(p || softmax(I)) over that set, gradient softmax(I) - p.
 *
 * Parity pins: tests/test_oracle_pins.py checks every function here against
 * brute force, closed forms, invariants and library routines.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------------- */
/* Number formats.                                                         */
/* ---------------------------------------------------------------------- */

/* FP8 E4M3 ("fn" variant: no infinities, 0x7F/0xFF are NaN): 1 sign bit,
 * 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 encodes the
 * subnormals m * 2^-9.  Decoded from the bit fields, not from a table copied
 * from anywhere. */
double oracle_e4m3_decode(uint8_t b) {
  int sign = (b >> 7) & 1;
  int e = (b >> 3) & 15;
  int m = b & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9); /* m/8 * 2^(1-7) */
  else
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

/* The e4m3 NaN codes (0x7F, 0xFF) are not values: an input that holds one is
 * an error of the caller, reported instead of scored.  Returns 1 if any of
 * the n bytes is such a code. */
static int has_e4m3_nan(const uint8_t* b, int64_t n) {
  for (int64_t i = 0; i < n; ++i)
    if ((b[i] & 0x7F) == 0x7F) return 1;
  return 0;
}

/* bfloat16 is the top half of an IEEE binary32. */
double oracle_bf16_decode(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* ---------------------------------------------------------------------- */
/* Lightning indexer.                                                       */
/* ---------------------------------------------------------------------- */

/* Score of query row i against key s (blog, "How the lightning indexer
 * works": weighted sum over indexer heads of ReLU(query-head . key)). */
static double indexer_score(const uint8_t* q8, const float* q_scale, const float* w,
                            const uint8_t* k8, const float* k_scale, int64_t i, int64_t s,
                            int H_I, int d_I) {
  double total = 0.0;
  for (int j = 0; j < H_I; ++j) {
    const uint8_t* qrow = q8 + ((int64_t)i * H_I + j) * d_I;
    const uint8_t* krow = k8 + (int64_t)s * d_I;
    double qs = (double)q_scale[(int64_t)i * H_I + j];
    double ks = (double)k_scale[s];
    double dot = 0.0;
    for (int d = 0; d < d_I; ++d)
      dot += (oracle_e4m3_decode(qrow[d]) * qs) * (oracle_e4m3_decode(krow[d]) * ks);
    double relu = dot > 0.0 ? dot : 0.0;
    total += (double)w[(int64_t)i * H_I + j] * relu;
  }
  return total;
}

/* For each listed local query row i (rows == NULL means rows 0..n_rows-1),
 * writes I[i, s] for s = 0..p_i into out[r * ld_out + s], p_i = n_k - n_q + i.
 * Entries s > p_i are left untouched.  Returns 0, or -1 on bad arguments. */
int oracle_indexer(const uint8_t* q8, const float* q_scale, const float* w, const uint8_t* k8,
                   const float* k_scale, int64_t n_q, int64_t n_k, int H_I, int d_I,
                   const int64_t* rows, int64_t n_rows, double* out, int64_t ld_out) {
  if (n_q < 0 || n_k < n_q || H_I <= 0 || d_I <= 0 || ld_out < n_k) return -1;
  if (has_e4m3_nan(q8, n_q * H_I * d_I) || has_e4m3_nan(k8, n_k * d_I)) return -2;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t i = rows ? rows[r] : r;
    if (i < 0 || i >= n_q) {
      bad = 1;
      continue;
    }
    int64_t p = n_k - n_q + i;
    for (int64_t s = 0; s <= p; ++s)
      out[r * ld_out + s] = indexer_score(q8, q_scale, w, k8, k_scale, i, s, H_I, d_I);
  }
  return bad ? -1 : 0;
}

/* ---------------------------------------------------------------------- */
/* Top-k selection.                                                         */
/* ---------------------------------------------------------------------- */

typedef struct {
  double v;
  int64_t s;
} scored_t;

/* Descending score, then ascending index.  -0.0 == +0.0 under IEEE compare,
 * so the two zeros are one value here. */
static int by_score_desc_index_asc(const void* a, const void* b) {
  const scored_t* x = (const scored_t*)a;
  const scored_t* y = (const scored_t*)b;
  if (x->v > y->v) return -1;
  if (x->v < y->v) return 1;
  return (x->s > y->s) - (x->s < y->s);
}

static int by_index_asc(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/* Selects, for one row of n = p + 1 candidate scores, the min(k, n) largest
 * by a full sort (blog, "How the lightning indexer works": a fixed number of
 * best-scoring entries is kept per query), writes them in ascending index order to idx[0..k) and pads with -1.
 * scratch holds at least n entries. */
static void topk_row(const double* scores, int64_t n, int k, scored_t* scratch, int32_t* idx) {
  for (int64_t s = 0; s < n; ++s) {
    double v = scores[s];
    if (v == 0.0) v = 0.0; /* -0 -> +0 */
    scratch[s].v = v;
    scratch[s].s = s;
  }
  qsort(scratch, (size_t)n, sizeof(scored_t), by_score_desc_index_asc);
  int64_t m = n < k ? n : k;
  for (int64_t r = 0; r < m; ++r) idx[r] = (int32_t)scratch[r].s;
  qsort(idx, (size_t)m, sizeof(int32_t), by_index_asc);
  for (int64_t r = m; r < k; ++r) idx[r] = -1;
}

/* scores: n_rows rows of stride ld; row r holds its candidates at 0..p_r,
 * p_r = n_k - n_q + rows[r].  idx_out: n_rows x k int32. */
int oracle_topk(const double* scores, int64_t ld, int64_t n_q, int64_t n_k, const int64_t* rows,
                int64_t n_rows, int k, int32_t* idx_out) {
  if (k <= 0 || n_k < n_q || ld < n_k) return -1;
  int bad = 0;
#pragma omp parallel
  {
    scored_t* scratch = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n_k > 0 ? n_k : 1));
#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < n_rows; ++r) {
      int64_t i = rows ? rows[r] : r;
      if (i < 0 || i >= n_q || !scratch) {
        bad = 1;
        continue;
      }
      int64_t p = n_k - n_q + i;
      topk_row(scores + r * ld, p + 1, k, scratch, idx_out + r * (int64_t)k);
    }
    free(scratch);
  }
  return bad ? -1 : 0;
}

/* ---------------------------------------------------------------------- */
/* Sparse attention, MQA mode of MLA.                                       */
/* ---------------------------------------------------------------------- */

/* One query row, all heads, over the selected set sel[0..n_sel).
 * Latent c[s] has d_qk dims; its first d_v dims are the value.  (blog, "How
 * the lightning indexer works": each latent is shared by all query heads.) */
static void attend_row(const uint16_t* q, const uint16_t* kv, const int32_t* sel, int64_t n_sel,
                       int64_t i, int H, int d_qk, int d_v, double scale, double* o, double* lse,
                       double* x) {
  for (int h = 0; h < H; ++h) {
    const uint16_t* qh = q + ((int64_t)i * H + h) * d_qk;
    double m = -INFINITY;
    for (int64_t r = 0; r < n_sel; ++r) {
      const uint16_t* c = kv + (int64_t)sel[r] * d_qk;
      double dot = 0.0;
      for (int d = 0; d < d_qk; ++d) dot += oracle_bf16_decode(qh[d]) * oracle_bf16_decode(c[d]);
      x[r] = scale * dot;
      if (x[r] > m) m = x[r];
    }
    double* oh = o + (int64_t)h * d_v;
    for (int d = 0; d < d_v; ++d) oh[d] = 0.0;
    double z = 0.0;
    for (int64_t r = 0; r < n_sel; ++r) {
      double e = exp(x[r] - m);
      z += e;
      const uint16_t* c = kv + (int64_t)sel[r] * d_qk;
      for (int d = 0; d < d_v; ++d) oh[d] += e * oracle_bf16_decode(c[d]);
    }
    if (n_sel == 0) {
      lse[h] = -INFINITY;
      continue;
    }
    for (int d = 0; d < d_v; ++d) oh[d] /= z;
    lse[h] = m + log(z);
  }
}

/* Keeps the entries of an index row that name a key the query may use
 * (0 <= s <= p), in row order. */
static int64_t valid_entries(const int32_t* idx_row, int k, int64_t p, int32_t* sel) {
  int64_t n = 0;
  for (int r = 0; r < k; ++r)
    if (idx_row[r] >= 0 && idx_row[r] <= p) sel[n++] = idx_row[r];
  return n;
}

/* q: n_q x H x d_qk bf16; kv: n_k x d_qk bf16; idx: n_rows x k (row r belongs
 * to local query rows[r]).  out: n_rows x H x d_v; lse: n_rows x H. */
int oracle_sparse_mla(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int64_t n_q,
                      int64_t n_k, int H, int d_qk, int d_v, int k, double scale,
                      const int64_t* rows, int64_t n_rows, double* out, double* lse) {
  if (k <= 0 || n_k < n_q || d_v > d_qk || H <= 0) return -1;
  int bad = 0;
#pragma omp parallel
  {
    int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    double* x = (double*)malloc(sizeof(double) * (size_t)k);
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
      int64_t i = rows ? rows[r] : r;
      if (i < 0 || i >= n_q || !sel || !x) {
        bad = 1;
        continue;
      }
      int64_t p = n_k - n_q + i;
      int64_t n_sel = valid_entries(idx + r * (int64_t)k, k, p, sel);
      attend_row(q, kv, sel, n_sel, i, H, d_qk, d_v, scale, out + r * (int64_t)H * d_v,
                 lse + r * (int64_t)H, x);
    }
    free(sel);
    free(x);
  }
  return bad ? -1 : 0;
}

/* ---------------------------------------------------------------------- */
/* The whole path for selected query rows.                                  */
/* ---------------------------------------------------------------------- */

/* indexer -> top-k -> sparse attention, one query row at a time.  idx_out
 * (n_rows x k), out (n_rows x H x d_v) and lse (n_rows x H) receive the
 * results; idx_out may be NULL. */
int oracle_forward(const uint8_t* q8, const float* q_scale, const float* w, const uint8_t* k8,
                   const float* k_scale, const uint16_t* q, const uint16_t* kv, int64_t n_q,
                   int64_t n_k, int H_I, int d_I, int H, int d_qk, int d_v, int k, double scale,
                   const int64_t* rows, int64_t n_rows, int32_t* idx_out, double* out,
                   double* lse) {
  if (k <= 0 || n_k < n_q || d_v > d_qk || H <= 0 || H_I <= 0 || d_I <= 0) return -1;
  if (has_e4m3_nan(q8, n_q * H_I * d_I) || has_e4m3_nan(k8, n_k * d_I)) return -2;
  int bad = 0;
#pragma omp parallel
  {
    double* scores = (double*)malloc(sizeof(double) * (size_t)(n_k > 0 ? n_k : 1));
    scored_t* scratch = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n_k > 0 ? n_k : 1));
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    double* x = (double*)malloc(sizeof(double) * (size_t)k);
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
      int64_t i = rows ? rows[r] : r;
      if (i < 0 || i >= n_q || !scores || !scratch || !idx || !sel || !x) {
        bad = 1;
        continue;
      }
      int64_t p = n_k - n_q + i;
      for (int64_t s = 0; s <= p; ++s)
        scores[s] = indexer_score(q8, q_scale, w, k8, k_scale, i, s, H_I, d_I);
      topk_row(scores, p + 1, k, scratch, idx);
      if (idx_out) memcpy(idx_out + r * (int64_t)k, idx, sizeof(int32_t) * (size_t)k);
      int64_t n_sel = valid_entries(idx, k, p, sel);
      attend_row(q, kv, sel, n_sel, i, H, d_qk, d_v, scale, out + r * (int64_t)H * d_v,
                 lse + r * (int64_t)H, x);
    }
    free(scores);
    free(scratch);
    free(idx);
    free(sel);
    free(x);
  }
  return bad ? -1 : 0;
}

/* The whole path for query rows given with their positions: row r of the
 * query-side arrays (q8, q_scale, w, q) sits at position pos[r] < n_k of a
 * sequence whose keys are k8 / k_scale / kv.  Same arithmetic as
 * oracle_forward; used to evaluate sampled rows of a long sequence without
 * materialising the other query rows. */
int oracle_forward_at(const uint8_t* q8, const float* q_scale, const float* w, const uint8_t* k8,
                      const float* k_scale, const uint16_t* q, const uint16_t* kv,
                      const int64_t* pos, int64_t n_rows, int64_t n_k, int H_I, int d_I, int H,
                      int d_qk, int d_v, int k, double scale, int32_t* idx_out, double* out,
                      double* lse) {
  if (k <= 0 || d_v > d_qk || H <= 0 || H_I <= 0 || d_I <= 0 || !pos) return -1;
  if (has_e4m3_nan(q8, n_rows * H_I * d_I) || has_e4m3_nan(k8, n_k * d_I)) return -2;
  int bad = 0;
#pragma omp parallel
  {
    double* scores = (double*)malloc(sizeof(double) * (size_t)(n_k > 0 ? n_k : 1));
    scored_t* scratch = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n_k > 0 ? n_k : 1));
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    double* x = (double*)malloc(sizeof(double) * (size_t)k);
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
      int64_t p = pos[r];
      if (p < 0 || p >= n_k || !scores || !scratch || !idx || !sel || !x) {
        bad = 1;
        continue;
      }
      for (int64_t s = 0; s <= p; ++s)
        scores[s] = indexer_score(q8, q_scale, w, k8, k_scale, r, s, H_I, d_I);
      topk_row(scores, p + 1, k, scratch, idx);
      if (idx_out) memcpy(idx_out + r * (int64_t)k, idx, sizeof(int32_t) * (size_t)k);
      int64_t n_sel = valid_entries(idx, k, p, sel);
      attend_row(q, kv, sel, n_sel, r, H, d_qk, d_v, scale, out + r * (int64_t)H * d_v,
                 lse + r * (int64_t)H, x);
    }
    free(scores);
    free(scratch);
    free(idx);
    free(sel);
    free(x);
  }
  return bad ? -1 : 0;
}

/* Indexer scores of query rows given with their positions: row r of q8 /
 * q_scale / w sits at position pos[r] < n_k; out[r * ld_out + s] = I[r, s]
 * for s <= pos[r]. */
int oracle_indexer_at(const uint8_t* q8, const float* q_scale, const float* w, const uint8_t* k8,
                      const float* k_scale, const int64_t* pos, int64_t n_rows, int64_t n_k,
                      int H_I, int d_I, double* out, int64_t ld_out) {
  if (H_I <= 0 || d_I <= 0 || ld_out < n_k || !pos) return -1;
  if (has_e4m3_nan(q8, n_rows * H_I * d_I) || has_e4m3_nan(k8, n_k * d_I)) return -2;
  for (int64_t r = 0; r < n_rows; ++r)
    if (pos[r] < 0 || pos[r] >= n_k) return -1;
  /* Few, long rows are the use of this entry (sampled rows of a long
   * sequence, decode rows), so the independent scores of a row are spread
   * over the host cores rather than the rows. */
  for (int64_t r = 0; r < n_rows; ++r) {
    const int64_t p = pos[r];
#pragma omp parallel for schedule(static)
    for (int64_t s = 0; s <= p; ++s)
      out[r * ld_out + s] = indexer_score(q8, q_scale, w, k8, k_scale, r, s, H_I, d_I);
  }
  return 0;
}

/* Sparse attention of query rows given with their positions (row r of q at
 * position pos[r]; idx row r is its selection). */
int oracle_sparse_mla_at(const uint16_t* q, const uint16_t* kv, const int32_t* idx,
                         const int64_t* pos, int64_t n_rows, int64_t n_k, int H, int d_qk,
                         int d_v, int k, double scale, double* out, double* lse) {
  if (k <= 0 || d_v > d_qk || H <= 0 || !pos) return -1;
  int bad = 0;
#pragma omp parallel
  {
    int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    double* x = (double*)malloc(sizeof(double) * (size_t)k);
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
      int64_t p = pos[r];
      if (p < 0 || p >= n_k || !sel || !x) {
        bad = 1;
        continue;
      }
      int64_t n_sel = valid_entries(idx + r * (int64_t)k, k, p, sel);
      attend_row(q, kv, sel, n_sel, r, H, d_qk, d_v, scale, out + r * (int64_t)H * d_v,
                 lse + r * (int64_t)H, x);
    }
    free(sel);
    free(x);
  }
  return bad ? -1 : 0;
}

/* ---------------------------------------------------------------------- */
/* Indexer training signal.                                                 */
/* ---------------------------------------------------------------------- */

/* KL alignment of the indexer to the main attention over the selected set
 * ("DeepSeek V3.2 and the lightning indexer", section "Teaching a dense model
 * to be sparse": the indexer's scores are fitted to the main attention's
 * distribution by minimising a KL divergence; "DeepSeek-V3.2" atlas entry,
 * "Design overview": the target is the head-wise attention distribution
 * summed over heads).  Readings: the target of query row r over its valid
 * selected entries S (the index row's entries 0 <= s <= p) is
 *     p[s] = (1/H) sum_h softmax_{s in S}(scale * q[r,h,:] . c[s,:]),
 * the indexer's distribution is q[s] = softmax_{s in S}(I[r, s]) of the given
 * scores, the loss is KL(p || q) = sum_s p[s] (log p[s] - log q[s]) and the
 * gradient of the loss with respect to I[r, s] is q[s] - p[s].
 * Row r of q is at position pos[r]; its scores are logits[r * ld + s].
 * Outputs per row: kl[r]; grad and target (nullable) n_rows x k in index-row
 * order, 0 at invalid entries.  The attention scores are taken afresh in fp64
 * (this function does not use the attention's lse). */
int oracle_indexer_kl_at(const uint16_t* q, const uint16_t* kv, const int32_t* idx,
                         const int64_t* pos, const float* logits, int64_t ld, int64_t n_rows,
                         int64_t n_k, int H, int d_qk, int k, double scale, double* kl,
                         double* grad, double* target) {
  if (k <= 0 || H <= 0 || !pos || !logits || !kl) return -1;
  int bad = 0;
#pragma omp parallel
  {
    int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    int32_t* slot = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    double* x = (double*)malloc(sizeof(double) * (size_t)k);
    double* pt = (double*)malloc(sizeof(double) * (size_t)k);
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
      const int64_t p = pos[r];
      if (p < 0 || p >= n_k || !sel || !slot || !x || !pt) {
        bad = 1;
        continue;
      }
      const int32_t* row = idx + r * (int64_t)k;
      int64_t n = 0;
      for (int j = 0; j < k; ++j)
        if (row[j] >= 0 && row[j] <= p) {
          sel[n] = row[j];
          slot[n] = j;
          ++n;
        }
      double* g = grad ? grad + r * (int64_t)k : NULL;
      double* tg = target ? target + r * (int64_t)k : NULL;
      for (int j = 0; j < k; ++j) {
        if (g) g[j] = 0.0;
        if (tg) tg[j] = 0.0;
      }
      if (n == 0) {
        kl[r] = 0.0;
        continue;
      }
      /* target: each head's softmax over S, averaged over the heads */
      for (int64_t e = 0; e < n; ++e) pt[e] = 0.0;
      for (int h = 0; h < H; ++h) {
        const uint16_t* qh = q + (r * H + h) * (int64_t)d_qk;
        double m = -INFINITY;
        for (int64_t e = 0; e < n; ++e) {
          const uint16_t* c = kv + (int64_t)sel[e] * d_qk;
          double dot = 0.0;
          for (int d = 0; d < d_qk; ++d) dot += oracle_bf16_decode(qh[d]) * oracle_bf16_decode(c[d]);
          x[e] = scale * dot;
          if (x[e] > m) m = x[e];
        }
        double z = 0.0;
        for (int64_t e = 0; e < n; ++e) z += exp(x[e] - m);
        for (int64_t e = 0; e < n; ++e) pt[e] += exp(x[e] - m) / z / (double)H;
      }
      /* the indexer's distribution: softmax of its scores over S */
      double mi = -INFINITY;
      for (int64_t e = 0; e < n; ++e) {
        x[e] = (double)logits[r * ld + sel[e]];
        if (x[e] > mi) mi = x[e];
      }
      double zi = 0.0;
      for (int64_t e = 0; e < n; ++e) zi += exp(x[e] - mi);
      const double log_zi = log(zi);
      double loss = 0.0;
      for (int64_t e = 0; e < n; ++e) {
        const double log_q = x[e] - mi - log_zi;
        if (pt[e] > 0.0) loss += pt[e] * (log(pt[e]) - log_q);
        if (g) g[slot[e]] = exp(log_q) - pt[e];
        if (tg) tg[slot[e]] = pt[e];
      }
      kl[r] = loss;
    }
    free(sel);
    free(slot);
    free(x);
    free(pt);
  }
  return bad ? -1 : 0;
}

/* The indexer's backward ("DeepSeek V3.2 and the lightning indexer", section
 * "Teaching a dense model to be sparse": in the dense warm-up only the
 * indexer learns, from the KL signal above).  Given the gradient g of a loss
 * with respect to the scores I[t,s] = sum_j w[t,j] * ReLU(q[t,j,:] . k[s,:])
 * (s <= p_t; q and k the dequantized FP8 values), the chain rule gives
 *     dw[t,j]   = sum_s g[t,s] * ReLU(q[t,j,:] . k[s,:])
 *     dq[t,j,:] = sum_s g[t,s] * w[t,j] * [q[t,j,:] . k[s,:] > 0] * k[s,:]
 *     dk[s,:]   = sum_t sum_j g[t,s] * w[t,j] * [q[t,j,:] . k[s,:] > 0] * q[t,j,:]
 * with the ReLU's derivative taken as 0 at 0.  Row t of q, w and g is at
 * position pos[t]; g is dense [n_q, n_k] and only s <= pos[t] is used.  q:
 * n_q x H x d; w: n_q x H; k: n_k x d; outputs dq (n_q x H x d), dw
 * (n_q x H), dk (n_k x d), all fp64.  dk sums over every row, so this runs
 * serially over rows. */
int oracle_indexer_backward(const double* q, const double* w, const double* k, const double* g,
                            const int64_t* pos, int64_t n_q, int64_t n_k, int H, int d,
                            double* dq, double* dw, double* dk) {
  if (!q || !w || !k || !g || !pos || !dq || !dw || !dk || H <= 0 || d <= 0) return -1;
  for (int64_t i = 0; i < n_q * H * d; ++i) dq[i] = 0.0;
  for (int64_t i = 0; i < n_q * H; ++i) dw[i] = 0.0;
  for (int64_t i = 0; i < n_k * d; ++i) dk[i] = 0.0;
  for (int64_t t = 0; t < n_q; ++t) {
    const int64_t p = pos[t];
    if (p < 0 || p >= n_k) return -1;
    for (int64_t s = 0; s <= p; ++s) {
      const double gs = g[t * n_k + s];
      if (gs == 0.0) continue;
      const double* ks = k + s * d;
      for (int j = 0; j < H; ++j) {
        const double* qj = q + (t * H + j) * d;
        double dot = 0.0;
        for (int e = 0; e < d; ++e) dot += qj[e] * ks[e];
        if (!(dot > 0.0)) continue;
        dw[t * H + j] += gs * dot;
        const double c = gs * w[t * H + j];
        double* dqj = dq + (t * H + j) * d;
        double* dks = dk + s * d;
        for (int e = 0; e < d; ++e) {
          dqj[e] += c * ks[e];
          dks[e] += c * qj[e];
        }
      }
    }
  }
  return 0;
}

/* ---------------------------------------------------------------------- */
/* Masked MHA mode.                                                         */
/* ---------------------------------------------------------------------- */

/* The masked MHA mode that stands in for DSA on short prefills ("DeepSeek-
 * V3.2" atlas entry, "Design overview" and "Inference efficiency" name it;
 * the pages give no detail).  Reading: dense attention
 * in the MHA form of MLA (every head has its own key and value), restricted
 * by a mask to the query's selected set S = { idx[r, j] : 0 <= idx[r, j] <= p }
 * taken as a set (a repeated entry counts once), keys visited in ascending
 * order:
 *     out[r,h,:] = sum_{s in S} softmax_s(scale * q[r,h,:] . k[s,h,:]) v[s,h,:]
 *     lse[r,h]   = log sum_{s in S} exp(scale * q[r,h,:] . k[s,h,:]).
 * q: n_rows x H x d_qk (row r at position pos[r]); k: n_k x H x d_qk;
 * v: n_k x H x d_v, all bf16 bits; idx: n_rows x topk.  A row with empty S
 * gets out = 0, lse = -inf. */
int oracle_masked_mha_at(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         const int32_t* idx, const int64_t* pos, int64_t n_rows, int64_t n_k,
                         int H, int d_qk, int d_v, int topk, double scale, double* out,
                         double* lse) {
  if (topk <= 0 || H <= 0 || d_qk <= 0 || d_v <= 0 || !pos || n_k <= 0) return -1;
  int bad = 0;
#pragma omp parallel
  {
    unsigned char* mark = (unsigned char*)calloc((size_t)n_k, 1);
    double* x = (double*)malloc(sizeof(double) * (size_t)n_k);
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
      const int64_t p = pos[r];
      if (p < 0 || p >= n_k || !mark || !x) {
        bad = 1;
        continue;
      }
      const int32_t* row = idx + r * (int64_t)topk;
      int64_t n_sel = 0;
      for (int j = 0; j < topk; ++j)
        if (row[j] >= 0 && row[j] <= p && !mark[row[j]]) {
          mark[row[j]] = 1;
          ++n_sel;
        }
      for (int h = 0; h < H; ++h) {
        const uint16_t* qh = q + (r * H + h) * (int64_t)d_qk;
        double* oh = out + (r * H + h) * (int64_t)d_v;
        for (int d = 0; d < d_v; ++d) oh[d] = 0.0;
        if (n_sel == 0) {
          lse[r * H + h] = -INFINITY;
          continue;
        }
        double m = -INFINITY;
        for (int64_t s = 0; s <= p; ++s) {
          if (!mark[s]) continue;
          const uint16_t* ks = k + (s * H + h) * (int64_t)d_qk;
          double dot = 0.0;
          for (int d = 0; d < d_qk; ++d) dot += oracle_bf16_decode(qh[d]) * oracle_bf16_decode(ks[d]);
          x[s] = scale * dot;
          if (x[s] > m) m = x[s];
        }
        double z = 0.0;
        for (int64_t s = 0; s <= p; ++s) {
          if (!mark[s]) continue;
          const double e = exp(x[s] - m);
          z += e;
          const uint16_t* vs = v + (s * H + h) * (int64_t)d_v;
          for (int d = 0; d < d_v; ++d) oh[d] += e * oracle_bf16_decode(vs[d]);
        }
        for (int d = 0; d < d_v; ++d) oh[d] /= z;
        lse[r * H + h] = m + log(z);
      }
      for (int j = 0; j < topk; ++j)
        if (row[j] >= 0 && row[j] <= p) mark[row[j]] = 0;
    }
    free(mark);
    free(x);
  }
  return bad ? -1 : 0;
}

/* Threads OpenMP will use (reported beside the CPU baseline). */
int oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
