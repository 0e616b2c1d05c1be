/*
 * dropkv_oracle.c -- plain fp64 CPU oracle for DropKV prefill-time eviction
 * scoring.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg call it; the product path never does.  It shares
 * no code, header or table with the CUDA library.
 *
 * What it computes, in the order the pages give it:
 *
 *   Window attention and single-removal perturbation -- write-up
 *   "DropKV：精确单项输出扰动评分组件", section 核心公式 (core formula):
 *       p = softmax(K q / sqrt(d)),  a = sum_j p_j v_j,
 *       Delta_j = p_j / (1 - p_j) * (a - v_j),
 *       s_j = sum over window queries t of ||Delta_j^(t)||_2^2.
 *   Causal tail alignment (same write-up, section 代码映射与边界): the last w
 *   prompt positions are the window queries; query t sits at position
 *   L - w + t and sees keys 0 .. L - w + t.
 *   GQA mean-merge (section 核心公式, the paragraph after the equation): the
 *   score of a physical KV head is the mean over the query heads that share
 *   it.  Query head hq maps to KV head hq / G (contiguous groups; the pages do
 *   not give the map, this is the standard grouped layout).
 *   Algorithm 1 (same paragraph): MaxPool1D over the token axis, then +inf on
 *   the final observation window, then evict the lowest scores.
 *   Singular input (same paragraph): a p_j that rounds to 1 makes exact
 *   removal undefined; it is rejected, with no epsilon.
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes): pooling kernel k odd, stride 1, window [j-k/2, j+k/2] clipped to
 * [0, L) (i.e. -inf padding); pooling runs over the merged scores of all of
 * [0, L) before the window is overwritten; positions >= L are NaN; "rounds to
 * 1" means the fp32 rounding of the exact p_j equals 1, or 1 - p_j is 0 in
 * fp64; eviction order is (score ascending, position ascending); keep and
 * evict lists are sorted by position and padded with -1.
 *
 * Everything is fp64, straight loops, one (batch, query head) per OpenMP
 * iteration.  No blocking, no fusion, no streaming.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_SINGULAR 2

static int check_shape(int B, int Hq, int Hkv, int n_max, int d, int w, int pool,
                       const int32_t* lengths) {
  if (B < 1 || Hq < 1 || Hkv < 1 || n_max < 1 || d < 1 || w < 1) return ORACLE_ERR_ARG;
  if (Hq % Hkv != 0) return ORACLE_ERR_ARG;
  if (pool < 1 || pool % 2 == 0) return ORACLE_ERR_ARG;
  for (int b = 0; b < B; ++b) {
    int L = lengths[b];
    if (L > n_max || L <= w) return ORACLE_ERR_ARG;
  }
  return ORACLE_OK;
}

/*
 * Window attention of one query over keys 0..P (core formula, first two
 * definitions).  Fills x (logits), p (probabilities), a (output, length d),
 * and returns the softmax normaliser through *l_out and the max through *m_out.
 */
static void window_attention(const double* q, const double* K, const double* V, int P, int d,
                             double* x, double* e, double* p, double* a, double* m_out,
                             double* l_out) {
  const double scale = 1.0 / sqrt((double)d);
  double m = -INFINITY;
  for (int j = 0; j <= P; ++j) {
    double dot = 0.0;
    for (int c = 0; c < d; ++c) dot += q[c] * K[(size_t)j * d + c];
    x[j] = dot * scale;
    if (x[j] > m) m = x[j];
  }
  double l = 0.0;
  for (int j = 0; j <= P; ++j) {
    e[j] = exp(x[j] - m);
    l += e[j];
  }
  for (int j = 0; j <= P; ++j) p[j] = e[j] / l;
  for (int c = 0; c < d; ++c) a[c] = 0.0;
  for (int j = 0; j <= P; ++j)
    for (int c = 0; c < d; ++c) a[c] += p[j] * V[(size_t)j * d + c];
  *m_out = m;
  *l_out = l;
}

/* "Rounds to 1": the fp32 rounding of p equals 1, or its complement is zero. */
static int is_singular(double p, double l, double e) {
  return ((float)p == 1.0f) || (l - e == 0.0);
}

/*
 * Per query head raw scores s[b, hq, j] (core formula, the s_j definition),
 * summed over the w window queries of that head.  Also returns each window
 * query's attention output and softmax statistics when asked.
 *
 * q:  [B, Hq, w, d]          k, v: [B, Hkv, n_max, d]   (row-major, fp64)
 * raw: [B, Hq, n_max]        attn_out: [B, Hq, w, d] or NULL
 * stats: [B, Hq, w, 2] = (max logit, normaliser) or NULL
 * singular_at: [4] = first (b, hq, t, j) found singular, or NULL
 */
int oracle_raw_scores(int B, int Hq, int Hkv, int n_max, int d, int w, const double* q,
                      const double* k, const double* v, const int32_t* lengths, double* raw,
                      double* attn_out, double* stats, int32_t* singular_at) {
  if (check_shape(B, Hq, Hkv, n_max, d, w, 1, lengths)) return ORACLE_ERR_ARG;
  const int G = Hq / Hkv;
  int status = ORACLE_OK;
  if (singular_at) singular_at[0] = singular_at[1] = singular_at[2] = singular_at[3] = -1;

#pragma omp parallel for schedule(dynamic, 1)
  for (int bh = 0; bh < B * Hq; ++bh) {
    const int b = bh / Hq, hq = bh % Hq, h = hq / G;
    const int L = lengths[b];
    const double* K = k + ((size_t)b * Hkv + h) * n_max * d;
    const double* V = v + ((size_t)b * Hkv + h) * n_max * d;
    double* s = raw + ((size_t)b * Hq + hq) * n_max;
    double* x = malloc(sizeof(double) * L);
    double* e = malloc(sizeof(double) * L);
    double* p = malloc(sizeof(double) * L);
    double* a = malloc(sizeof(double) * d);
    for (int j = 0; j < n_max; ++j) s[j] = (j < L) ? 0.0 : NAN;
    for (int t = 0; t < w; ++t) {
      const int P = L - w + t; /* causal tail alignment */
      const double* qt = q + (((size_t)b * Hq + hq) * w + t) * d;
      double m, l;
      window_attention(qt, K, V, P, d, x, e, p, a, &m, &l);
      if (attn_out) memcpy(attn_out + (((size_t)b * Hq + hq) * w + t) * d, a, sizeof(double) * d);
      if (stats) {
        stats[(((size_t)b * Hq + hq) * w + t) * 2 + 0] = m;
        stats[(((size_t)b * Hq + hq) * w + t) * 2 + 1] = l;
      }
      for (int j = 0; j <= P; ++j) {
        if (is_singular(p[j], l, e[j])) {
#pragma omp critical
          {
            if (status == ORACLE_OK && singular_at) {
              singular_at[0] = b; singular_at[1] = hq; singular_at[2] = t; singular_at[3] = j;
            }
            status = ORACLE_ERR_SINGULAR;
          }
          continue;
        }
        /* Delta_j = p_j / (1 - p_j) (a - v_j); add its squared norm. */
        const double ratio = p[j] / (1.0 - p[j]);
        double sq = 0.0;
        for (int c = 0; c < d; ++c) {
          const double diff = ratio * (a[c] - V[(size_t)j * d + c]);
          sq += diff * diff;
        }
        s[j] += sq;
      }
    }
    free(x); free(e); free(p); free(a);
  }
  return status;
}

/*
 * Attention-only score, the negative control of the write-up
 * "DropKV：精确单项输出扰动评分组件", section 结果与独立对照: the pages name an
 * "attention-only" control beside the perturbation score without defining
 * it; the reading taken here is the plainest one, the attention mass each
 * token receives from the window queries,
 *     raw[b, hq, j] = sum over window queries t with j <= P_t of p_j^(t),
 * passed through the same merge / pool / protect / select as the perturbation
 * score.  Nothing is singular here.  Padding positions are NaN.
 */
int oracle_attn_raw(int B, int Hq, int Hkv, int n_max, int d, int w, const double* q,
                    const double* k, const int32_t* lengths, double* raw) {
  if (check_shape(B, Hq, Hkv, n_max, d, w, 1, lengths)) return ORACLE_ERR_ARG;
  const int G = Hq / Hkv;

#pragma omp parallel for schedule(dynamic, 1)
  for (int bh = 0; bh < B * Hq; ++bh) {
    const int b = bh / Hq, hq = bh % Hq, h = hq / G;
    const int L = lengths[b];
    const double* K = k + ((size_t)b * Hkv + h) * n_max * d;
    double* s = raw + ((size_t)b * Hq + hq) * n_max;
    double* x = malloc(sizeof(double) * L);
    for (int j = 0; j < n_max; ++j) s[j] = (j < L) ? 0.0 : NAN;
    for (int t = 0; t < w; ++t) {
      const int P = L - w + t; /* causal tail alignment */
      const double* qt = q + (((size_t)b * Hq + hq) * w + t) * d;
      /* p = softmax over keys 0..P of q.k / sqrt(d) */
      double m = -INFINITY;
      for (int j = 0; j <= P; ++j) {
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += qt[c] * K[(size_t)j * d + c];
        x[j] = dot / sqrt((double)d);
        if (x[j] > m) m = x[j];
      }
      double l = 0.0;
      for (int j = 0; j <= P; ++j) l += exp(x[j] - m);
      for (int j = 0; j <= P; ++j) s[j] += exp(x[j] - m) / l;
    }
    free(x);
  }
  return ORACLE_OK;
}

/* GQA mean-merge: merged[b, h, j] = mean over g of raw[b, h*G + g, j]. */
void oracle_merge(int B, int Hq, int Hkv, int n_max, const double* raw, const int32_t* lengths,
                  double* merged) {
  const int G = Hq / Hkv;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hkv; ++h)
      for (int j = 0; j < n_max; ++j) {
        double* out = merged + ((size_t)b * Hkv + h) * n_max + j;
        if (j >= lengths[b]) { *out = NAN; continue; }
        double sum = 0.0;
        for (int g = 0; g < G; ++g) sum += raw[((size_t)b * Hq + h * G + g) * n_max + j];
        *out = sum / G;
      }
}

/* MaxPool1D (odd kernel, stride 1, window clipped to [0, L)), then +inf on
 * the last w positions; NaN beyond the length. */
void oracle_pool_protect(int B, int Hkv, int n_max, int w, int pool, const double* merged,
                         const int32_t* lengths, double* scores) {
  const int r = pool / 2;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hkv; ++h) {
      const int L = lengths[b];
      const double* in = merged + ((size_t)b * Hkv + h) * n_max;
      double* out = scores + ((size_t)b * Hkv + h) * n_max;
      for (int j = 0; j < n_max; ++j) {
        if (j >= L) { out[j] = NAN; continue; }
        if (j >= L - w) { out[j] = INFINITY; continue; }
        double best = -INFINITY;
        for (int i = j - r; i <= j + r; ++i)
          if (i >= 0 && i < L && in[i] > best) best = in[i];
        out[j] = best;
      }
    }
}

/* The whole scoring path: raw -> merge -> pool -> protect. */
int oracle_scores(int B, int Hq, int Hkv, int n_max, int d, int w, int pool, const double* q,
                  const double* k, const double* v, const int32_t* lengths, double* scores,
                  double* merged_out, double* raw_out, double* attn_out, double* stats,
                  int32_t* singular_at) {
  if (check_shape(B, Hq, Hkv, n_max, d, w, pool, lengths)) return ORACLE_ERR_ARG;
  double* raw = raw_out ? raw_out : malloc(sizeof(double) * (size_t)B * Hq * n_max);
  double* merged = merged_out ? merged_out : malloc(sizeof(double) * (size_t)B * Hkv * n_max);
  int st = oracle_raw_scores(B, Hq, Hkv, n_max, d, w, q, k, v, lengths, raw, attn_out, stats,
                             singular_at);
  oracle_merge(B, Hq, Hkv, n_max, raw, lengths, merged);
  oracle_pool_protect(B, Hkv, n_max, w, pool, merged, lengths, scores);
  if (!raw_out) free(raw);
  if (!merged_out) free(merged);
  return st;
}

/*
 * Final scores at selected positions of one KV head, for inputs too large to
 * score whole.  K, V: [L, d] of that head; Qg: [G, w, d] of its query group.
 * For every window query the full attention row is computed, then only the
 * positions inside the pooling neighbourhoods of the requested ones are scored.
 */
int oracle_scores_at(int G, int L, int d, int w, int pool, const double* Qg, const double* K,
                     const double* V, int npos, const int32_t* pos, double* out) {
  if (G < 1 || d < 1 || w < 1 || L <= w || pool < 1 || pool % 2 == 0) return ORACLE_ERR_ARG;
  const int r = pool / 2;
  char* need = calloc((size_t)L, 1);
  for (int i = 0; i < npos; ++i) {
    if (pos[i] < 0 || pos[i] >= L) { free(need); return ORACLE_ERR_ARG; }
    for (int j = pos[i] - r; j <= pos[i] + r; ++j)
      if (j >= 0 && j < L) need[j] = 1;
  }
  int nneed = 0;
  for (int j = 0; j < L; ++j) nneed += need[j];
  int32_t* list = malloc(sizeof(int32_t) * (nneed ? nneed : 1));
  nneed = 0;
  for (int j = 0; j < L; ++j) if (need[j]) list[nneed++] = j;
  double* merged = calloc((size_t)L, sizeof(double));
  int status = ORACLE_OK;

#pragma omp parallel
  {
    double* x = malloc(sizeof(double) * L);
    double* e = malloc(sizeof(double) * L);
    double* p = malloc(sizeof(double) * L);
    double* a = malloc(sizeof(double) * d);
    double* acc = calloc((size_t)(nneed ? nneed : 1), sizeof(double));
#pragma omp for schedule(dynamic, 1)
    for (int gt = 0; gt < G * w; ++gt) {
      const int t = gt % w;
      const int P = L - w + t;
      double m, l;
      window_attention(Qg + (size_t)gt * d, K, V, P, d, x, e, p, a, &m, &l);
      for (int i = 0; i < nneed; ++i) {
        const int j = list[i];
        if (j > P) continue;
        if (is_singular(p[j], l, e[j])) {
#pragma omp atomic write
          status = ORACLE_ERR_SINGULAR;
          continue;
        }
        const double ratio = p[j] / (1.0 - p[j]);
        double sq = 0.0;
        for (int c = 0; c < d; ++c) {
          const double diff = ratio * (a[c] - V[(size_t)j * d + c]);
          sq += diff * diff;
        }
        acc[i] += sq;
      }
    }
#pragma omp critical
    for (int i = 0; i < nneed; ++i) merged[list[i]] += acc[i];
    free(x); free(e); free(p); free(a); free(acc);
  }
  for (int i = 0; i < nneed; ++i) merged[list[i]] /= G;
  for (int i = 0; i < npos; ++i) {
    const int j = pos[i];
    if (j >= L - w) { out[i] = INFINITY; continue; }
    double best = -INFINITY;
    for (int u = j - r; u <= j + r; ++u)
      if (u >= 0 && u < L && merged[u] > best) best = merged[u];
    out[i] = best;
  }
  free(need); free(list); free(merged);
  return status;
}

/* ---- selection: evict the lowest scores (Algorithm 1's last step) ---- */

typedef struct { double s; int32_t j; } keyed;

/* Order: score ascending, then position ascending; NaN above everything. */
static int cmp_keyed(const void* A, const void* Bp) {
  const keyed* a = (const keyed*)A;
  const keyed* b = (const keyed*)Bp;
  const int an = isnan(a->s), bn = isnan(b->s);
  if (an != bn) return an - bn;
  if (!an) {
    if (a->s < b->s) return -1;
    if (a->s > b->s) return 1;
  }
  return (a->j > b->j) - (a->j < b->j);
}

static int cmp_i32(const void* A, const void* Bp) {
  const int32_t a = *(const int32_t*)A, b = *(const int32_t*)Bp;
  return (a > b) - (a < b);
}

/*
 * For each (b, h): evict the lengths[b] - keep[b] lowest-ordered positions of
 * scores[b, h, 0:L].  keep_idx: [B, Hkv, max_keep], evict_idx: [B, Hkv,
 * max_evict], each sorted by position and padded with -1.
 */
int oracle_select(int B, int Hkv, int n_max, const double* scores, const int32_t* lengths,
                  const int32_t* keep, int max_keep, int max_evict, int32_t* keep_idx,
                  int32_t* evict_idx) {
  for (int b = 0; b < B; ++b) {
    const int L = lengths[b];
    if (L < 0 || L > n_max || keep[b] < 0 || keep[b] > L) return ORACLE_ERR_ARG;
    if (keep[b] > max_keep || L - keep[b] > max_evict) return ORACLE_ERR_ARG;
  }
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hkv; ++h) {
      const int L = lengths[b], E = L - keep[b];
      const double* s = scores + ((size_t)b * Hkv + h) * n_max;
      keyed* arr = malloc(sizeof(keyed) * (L ? L : 1));
      for (int j = 0; j < L; ++j) { arr[j].s = s[j]; arr[j].j = j; }
      qsort(arr, (size_t)L, sizeof(keyed), cmp_keyed);
      int32_t* ev = evict_idx + ((size_t)b * Hkv + h) * max_evict;
      int32_t* kp = keep_idx + ((size_t)b * Hkv + h) * max_keep;
      for (int i = 0; i < max_evict; ++i) ev[i] = -1;
      for (int i = 0; i < max_keep; ++i) kp[i] = -1;
      for (int i = 0; i < E; ++i) ev[i] = arr[i].j;
      for (int i = E; i < L; ++i) kp[i - E] = arr[i].j;
      qsort(ev, (size_t)E, sizeof(int32_t), cmp_i32);
      qsort(kp, (size_t)(L - E), sizeof(int32_t), cmp_i32);
      free(arr);
    }
  return ORACLE_OK;
}
