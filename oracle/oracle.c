/*
 * CPU oracle for modality-aware permutation sparse attention (MMInference,
 * ICML 2025) and the dynamic sparse patterns it inherits from MInference 1.0
 * (NeurIPS 2024).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links or calls this
 * file: it is the slow, plain, obviously-correct statement of what the path
 * computes, used by the tests, by smoke() and by the timed CPU baseline.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * Precision: bf16 inputs are widened exactly; every dot product is accumulated
 * in fp64 and rounded to fp32 (the precision of an fp32-accumulating tensor-core
 * logit), then multiplied by the fp32 softmax scale.  Softmax, probability sums
 * and the attention output are accumulated in fp64.
 *
 * Every function is deterministic: parallel loops only ever partition outputs,
 * never the terms of one sum.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static inline double bf(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* logit of query q against key k: fp32(sum_c q_c k_c) * scale, fp32 throughout */
static inline float logit(const uint16_t* q, const uint16_t* k, int d, float scale) {
  double acc = 0.0;
  for (int c = 0; c < d; ++c) acc += bf(q[c]) * bf(k[c]);
  float x = (float)acc;
  return x * scale;
}

/*
 * Last-query attention sums (MInference 1.0, section "Approach": vertical and
 * slash lines come from the attention rows of the final 64 queries; MMInference,
 * "core discovery": video-aware heads take those 64 rows per modality).
 *
 * For each estimation row r (original position rows[r]) the causal softmax
 * A[r, j] = exp(x_rj - m_r) / Z_r over all keys j <= rows[r] is formed, and
 *   v[j] += A[r, j]                                   (vertical / column sum)
 *   s[rcoord[r] - kcoord[j]] += A[r, j]  if kcoord[j] >= 0 and the offset >= 0
 * (slash / diagonal sum in a coordinate system given per row and per key:
 * original positions for vertical-slash and Q-boundary heads, within-modality
 * ranks for 2D-boundary heads).  v and s have length L and are zeroed here.
 */
void orc_lastq_sums(const uint16_t* Qh, const uint16_t* Kh, int64_t L, int d, float scale,
                    const int64_t* rows, int n_rows, const int64_t* rcoord, const int64_t* kcoord,
                    double* v, double* s) {
  memset(v, 0, sizeof(double) * (size_t)L);
  memset(s, 0, sizeof(double) * (size_t)L);
  float* x = (float*)malloc(sizeof(float) * (size_t)L);
  double* e = (double*)malloc(sizeof(double) * (size_t)L);
  for (int r = 0; r < n_rows; ++r) {
    const int64_t i = rows[r];
    const uint16_t* q = Qh + (size_t)i * d;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j <= i; ++j) x[j] = logit(q, Kh + (size_t)j * d, d, scale);
    double m = -INFINITY;
    for (int64_t j = 0; j <= i; ++j) m = x[j] > m ? x[j] : m;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j <= i; ++j) e[j] = exp((double)x[j] - m);
    double Z = 0.0;
    for (int64_t j = 0; j <= i; ++j) Z += e[j];
    const int64_t rc = rcoord[r];
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j <= i; ++j) {
      double a = e[j] / Z;
      v[j] += a;
      if (kcoord[j] >= 0) {
        int64_t o = rc - kcoord[j];
        if (o >= 0 && o < L) s[o] += a; /* o -> j is one-to-one for a fixed row */
      }
    }
  }
  free(x);
  free(e);
}

/*
 * Top-k selection.  Scores are rounded to fp32 (the precision the kernels take
 * the decision in), candidates are ordered by (score descending, index
 * ascending) and the first k are returned sorted by index.  Returns the number
 * written: min(k, number of candidates).  cand may be NULL (all candidates).
 */
typedef struct {
  float key;
  int64_t idx;
} orc_item;

static int cmp_item(const void* a, const void* b) {
  const orc_item* x = (const orc_item*)a;
  const orc_item* y = (const orc_item*)b;
  if (x->key != y->key) return x->key > y->key ? -1 : 1;
  return x->idx < y->idx ? -1 : (x->idx > y->idx ? 1 : 0);
}

static int cmp_i64(const void* a, const void* b) {
  int64_t x = *(const int64_t*)a, y = *(const int64_t*)b;
  return x < y ? -1 : (x > y ? 1 : 0);
}

int64_t orc_topk(const double* score, const uint8_t* cand, int64_t n, int64_t k, int64_t* out) {
  orc_item* it = (orc_item*)malloc(sizeof(orc_item) * (size_t)(n > 0 ? n : 1));
  int64_t m = 0;
  for (int64_t j = 0; j < n; ++j) {
    if (cand && !cand[j]) continue;
    it[m].key = (float)score[j];
    it[m].idx = j;
    ++m;
  }
  qsort(it, (size_t)m, sizeof(orc_item), cmp_item);
  int64_t c = k < m ? k : m;
  for (int64_t t = 0; t < c; ++t) out[t] = it[t].idx;
  qsort(out, (size_t)c, sizeof(int64_t), cmp_i64);
  free(it);
  return c;
}

/*
 * Mean pooling over blocks of 64 tokens (MInference 1.0, "Approach": block-sparse
 * heads estimate their index from mean-pooled 64-token blocks of Q and K).
 * out[b][c] = (1/64) * sum_{t in block b} X[t][c], fp64.
 */
void orc_pool64(const uint16_t* Xh, int64_t L, int d, double* out) {
  const int64_t nb = L / 64;
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < nb; ++b) {
    for (int c = 0; c < d; ++c) {
      double acc = 0.0;
      for (int t = 0; t < 64; ++t) acc += bf(Xh[(size_t)(b * 64 + t) * d + c]);
      out[b * d + c] = acc / 64.0;
    }
  }
}

/*
 * Block-sparse index: for query block b the candidates are key blocks c <= b,
 * scored by the pooled logit  Qbar_b . Kbar_c * scale  (fp64, decided in fp32);
 * softmax over a row is monotone, so the top-k of the logits is the top-k of the
 * pooled attention.  kk[b] blocks are kept (clipped to b + 1); out is [nb][kmax]
 * with counts[b] entries used, sorted ascending.
 */
void orc_block_topk(const double* Qbar, const double* Kbar, int64_t nb, int d, float scale,
                    const int64_t* kk, int64_t kmax, int64_t* out, int64_t* counts) {
#pragma omp parallel
  {
    double* sc = (double*)malloc(sizeof(double) * (size_t)nb);
#pragma omp for schedule(dynamic, 4)
    for (int64_t b = 0; b < nb; ++b) {
      for (int64_t c = 0; c <= b; ++c) {
        double acc = 0.0;
        for (int t = 0; t < d; ++t) acc += Qbar[b * d + t] * Kbar[c * d + t];
        sc[c] = acc * (double)scale;
      }
      int64_t k = kk[b] < b + 1 ? kk[b] : b + 1;
      if (k > kmax) k = kmax;
      counts[b] = orc_topk(sc, NULL, b + 1, k, out + b * kmax);
    }
    free(sc);
  }
}

/* ---------------------------------------------------------------------------------- */
/* token-level masks                                                                   */
/* ---------------------------------------------------------------------------------- */
enum { K_DENSE = 0, K_ASHAPE = 1, K_VSLASH = 2, K_BLOCK = 3, K_GRID = 4, K_QBOUND = 5, K_BOUND2D = 6, K_QSEG = 7 };

typedef struct {
  int32_t kind;
  int32_t _pad;
  int64_t sink;  /* A-shape sink tokens */
  int64_t local; /* A-shape local window; grid local band */
  /* vertical lines: vcol[a*2+b][j] != 0 marks key j for queries of modality a and
     keys of modality b (vertical-slash: only [0] is used, for every query;
     Q-boundary: [a*2+0] holds modality a's lines over all keys) */
  const uint8_t* vcol[4];
  /* slash lines: slash[a][o] != 0 marks offset o for queries of modality a */
  const uint8_t* slash[2];
  const uint8_t* gmark;    /* grid: tokens on the selected (stride, phase) lines */
  const uint8_t* modality; /* 0 text, 1 video */
  const int64_t* rank;     /* rank of a token among the tokens of its modality */
  const uint8_t* blocksel; /* block-sparse: [nb][nb] selected (query block, key block) */
  int64_t nb;
  /* Q-boundary estimated per segment: segid[t] = segment of token t; vseg[k] / sseg[k] mark the
     vertical keys / slash offsets estimated for the queries of segment k */
  const int32_t* segid;
  const uint8_t* const* vseg;
  const uint8_t* const* sseg;
} orc_mask;

/*
 * allowed(i, j): the sparse pattern of one head, ANDed with causality j <= i.
 *  A-shape (StreamingLLM-derived, MInference 1.0 "Approach"): sink or local window.
 *  Vertical-slash (MInference 1.0): key on a vertical line, or offset i-j on a slash line.
 *  Block-sparse (MInference 1.0): the 64-token (query block, key block) pair was selected.
 *  Grid (MMInference Algorithm 1, "key machinery"): video queries and keys on the
 *    selected horizontal/vertical grid lines, text queries, plus a local band.
 *  Q-boundary (MMInference Algorithm 2): vertical-slash per query modality; estimated per
 *    modality segment, vertical-slash per query segment (the queries of segment k use the
 *    lines estimated from segment k's last 64 queries).
 *  2D-boundary (MMInference Algorithm 3): per (query modality, key modality) pair;
 *    intra-modality pairs are vertical-slash in within-modality (compacted)
 *    coordinates, so slash lines continue across text-interrupted video;
 *    cross-modality pairs keep vertical lines only.
 */
static inline int allowed(const orc_mask* m, int64_t i, int64_t j) {
  if (j > i) return 0;
  switch (m->kind) {
    case K_DENSE:
      return 1;
    case K_ASHAPE:
      return j < m->sink || i - j < m->local;
    case K_VSLASH:
      return m->vcol[0][j] || m->slash[0][i - j];
    case K_BLOCK:
      return m->blocksel[(i / 64) * m->nb + j / 64] != 0;
    case K_GRID:
      return m->gmark[i] || m->modality[i] == 0 || m->gmark[j] || i - j < m->local;
    case K_QBOUND: {
      int a = m->modality[i];
      return m->vcol[a * 2][j] || m->slash[a][i - j];
    }
    case K_BOUND2D: {
      int a = m->modality[i], b = m->modality[j];
      if (a == b) return m->vcol[a * 2 + a][j] || m->slash[a][m->rank[i] - m->rank[j]];
      return m->vcol[a * 2 + b][j] != 0;
    }
    case K_QSEG: {
      const int32_t k = m->segid[i];
      return m->vseg[k][j] || m->sseg[k][i - j];
    }
  }
  return 0;
}

/* Dense 0/1 mask of the given rows (for small L): out[r][j] = allowed(rows[r], j). */
void orc_mask_rows(const orc_mask* m, int64_t L, const int64_t* rows, int64_t n_rows, uint8_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n_rows; ++r)
    for (int64_t j = 0; j < L; ++j) out[r * L + j] = (uint8_t)allowed(m, rows[r], j);
}

/* Number of allowed (i, j) pairs in each of the given rows. */
void orc_mask_count(const orc_mask* m, const int64_t* rows, int64_t n_rows, int64_t* out) {
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t c = 0;
    for (int64_t j = 0; j <= rows[r]; ++j) c += allowed(m, rows[r], j);
    out[r] = c;
  }
}

/*
 * Masked causal softmax attention for the given query rows of one head
 * (FlashAttention-style kernels compute exactly this; the oracle takes it
 * directly, row by row, visiting only allowed keys):
 *   O[r] = sum_j p_j V[j] / sum_j p_j,  p_j = exp(x_j - max_j x_j),  j allowed
 *   lse[r] = max_j x_j + log(sum_j p_j)      (natural log, logits x = q.k*scale)
 * A row with no allowed key gets O = 0 and lse = -inf.
 */
void orc_attention(const uint16_t* Qh, const uint16_t* Kh, const uint16_t* Vh, int64_t L, int d,
                   float scale, const orc_mask* m, const int64_t* rows, int64_t n_rows, float* O,
                   float* lse) {
#pragma omp parallel
  {
    float* x = (float*)malloc(sizeof(float) * (size_t)L);
    int64_t* js = (int64_t*)malloc(sizeof(int64_t) * (size_t)L);
    double* acc = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 8)
    for (int64_t r = 0; r < n_rows; ++r) {
      const int64_t i = rows[r];
      const uint16_t* q = Qh + (size_t)i * d;
      int64_t n = 0;
      float mx = -INFINITY;
      for (int64_t j = 0; j <= i; ++j) {
        if (!allowed(m, i, j)) continue;
        js[n] = j;
        x[n] = logit(q, Kh + (size_t)j * d, d, scale);
        if (x[n] > mx) mx = x[n];
        ++n;
      }
      if (n == 0) {
        for (int c = 0; c < d; ++c) O[r * d + c] = 0.0f;
        lse[r] = -INFINITY;
        continue;
      }
      for (int c = 0; c < d; ++c) acc[c] = 0.0;
      double Z = 0.0;
      for (int64_t t = 0; t < n; ++t) {
        double p = exp((double)x[t] - (double)mx);
        Z += p;
        const uint16_t* vr = Vh + (size_t)js[t] * d;
        for (int c = 0; c < d; ++c) acc[c] += p * bf(vr[c]);
      }
      for (int c = 0; c < d; ++c) O[r * d + c] = (float)(acc[c] / Z);
      lse[r] = (float)((double)mx + log(Z));
    }
    free(x);
    free(js);
    free(acc);
  }
}

/*
 * Masked attention taken in permuted coordinates (MMInference review page, "core
 * discovery": the permutation is realised as index-based loading, so the output of a
 * head does not change; "key machinery": grid, Q-boundary and 2D-boundary heads
 * permute the query and key axes so that the selected entries become contiguous).
 *
 * Row r of Qp is the query at original position qpos[r]; row t of Kp and Vp is the key
 * at original position kpos[t].  Causality and the head's pattern are evaluated
 * through the original positions, allowed(qpos[r], kpos[t]); the keys are visited in
 * permuted order t = 0 .. nk - 1.  Output row r (and lse[r]) belongs to original
 * position qpos[r]: the caller scatters it back.  Same arithmetic as orc_attention
 * except for the order of the fp64 sums.
 */
void orc_attention_permuted(const uint16_t* Qp, const uint16_t* Kp, const uint16_t* Vp,
                            const int64_t* qpos, int64_t nq, const int64_t* kpos, int64_t nk, int d,
                            float scale, const orc_mask* m, float* Op, float* lse) {
#pragma omp parallel
  {
    float* x = (float*)malloc(sizeof(float) * (size_t)(nk > 0 ? nk : 1));
    int64_t* ts = (int64_t*)malloc(sizeof(int64_t) * (size_t)(nk > 0 ? nk : 1));
    double* acc = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 8)
    for (int64_t r = 0; r < nq; ++r) {
      const int64_t i = qpos[r];
      const uint16_t* q = Qp + (size_t)r * d;
      int64_t n = 0;
      float mx = -INFINITY;
      for (int64_t t = 0; t < nk; ++t) {
        if (!allowed(m, i, kpos[t])) continue;
        ts[n] = t;
        x[n] = logit(q, Kp + (size_t)t * d, d, scale);
        if (x[n] > mx) mx = x[n];
        ++n;
      }
      if (n == 0) {
        for (int c = 0; c < d; ++c) Op[r * d + c] = 0.0f;
        lse[r] = -INFINITY;
        continue;
      }
      for (int c = 0; c < d; ++c) acc[c] = 0.0;
      double Z = 0.0;
      for (int64_t u = 0; u < n; ++u) {
        double p = exp((double)x[u] - (double)mx);
        Z += p;
        const uint16_t* vr = Vp + (size_t)ts[u] * d;
        for (int c = 0; c < d; ++c) acc[c] += p * bf(vr[c]);
      }
      for (int c = 0; c < d; ++c) Op[r * d + c] = (float)(acc[c] / Z);
      lse[r] = (float)((double)mx + log(Z));
    }
    free(x);
    free(ts);
    free(acc);
  }
}
