/*
 * CPU oracle for the DeepSeek Sparse Attention lightning-indexer hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: it exists so that tests, the smoke check and the timed CPU
 * baseline can compare the CUDA library against a plain, slow, obviously
 * correct restatement of the method.  It shares no code with the CUDA path.
 *
 * Everything is computed in fp64 from the exact input bits: bf16 q/k values
 * and fp32 head weights widen to fp64 without rounding.
 *
 * Sources (page title, section / equation):
 *  - "DeepSeek DSA FLOPs", Lightning Indexer, eq. (index score):
 *        I(t,s) = sum_j w(t,j) * ReLU(q(t,j) . k(s))
 *  - "DeepSeek DSA FLOPs", causal token-pair count: query at 0-based position
 *    p sees keys 0..p (N_dense = T(T+1)/2), and keeps m = min(k, p+1) of them
 *    (N_sel).
 *  - "计算DSA的时间复杂度", step 3: Top-k is a selection of the k largest scores.
 *  - "DoSA: Dots Sparse Attention：阅读材料", annotation LBKERZAW (steps 1-3)
 *    and the 163.com write-up, section 03: seed threshold, per-key upper
 *    bound from retained heads + positive residual bound + folded negative
 *    heads, strict pruning, exact refine, final selection by full score.
 *
 * Readings where the pages are silent: ties in Top-k are broken by the
 * smaller key index; rows with fewer than k visible keys are padded with
 * index -1 and score -inf; the weights are used as given (no extra scale).
 *
 * Pins: every function here is checked by tests/test_oracle_pins.py against
 * something other than itself: the worked numbers "DeepSeek DSA FLOPs"
 * prints, a hand-worked example, reductions to a textbook matmul + sort
 * (numpy), linearity and homogeneity, exhaustive selection on tiny inputs,
 * the planner sample positions the DoSA notes print, and DoSA cases where the
 * bound is exact or must hold.  oracle_score_pairs is pinned against a numpy
 * matmul of the widened inputs at random (row, key) pairs of chunked and
 * decode layouts.  Parity is unpinned only for the per-element fp32 results
 * of the GPU beyond the stated tolerance.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_API __attribute__((visibility("default")))

static inline double bf16_to_f64(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* ---------------------------------------------------------------------------
 * Index score, written out as the definition (eq. index score).
 * ------------------------------------------------------------------------ */
static double dot_f64(const uint16_t *a, const uint16_t *b, int d) {
  double acc = 0.0;
  for (int i = 0; i < d; ++i) acc += bf16_to_f64(a[i]) * bf16_to_f64(b[i]);
  return acc;
}

static double index_score(const uint16_t *q_row, const float *w_row,
                          const uint16_t *k_s, int H, int d) {
  double I = 0.0;
  for (int j = 0; j < H; ++j) {
    double x = dot_f64(q_row + (size_t)j * d, k_s, d);
    double relu = x > 0.0 ? x : 0.0;
    I += (double)w_row[j] * relu;
  }
  return I;
}

/* I(t, s) for s in [0, n_keys). */
OR_API void oracle_row_scores(const uint16_t *q_row, const float *w_row,
                              const uint16_t *k, int64_t n_keys, int H, int d,
                              double *out) {
  for (int64_t s = 0; s < n_keys; ++s)
    out[s] = index_score(q_row, w_row, k + (size_t)s * d, H, d);
}

/* Scores of arbitrary (query row, key) pairs: q_rows[n] indexes q/w rows. */
OR_API void oracle_score_pairs(const uint16_t *q, const float *w,
                               const uint16_t *k, int H, int d, int64_t n,
                               const int64_t *q_rows, const int64_t *keys,
                               double *out, int n_threads) {
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 64)
#endif
  for (int64_t i = 0; i < n; ++i)
    out[i] = index_score(q + (size_t)q_rows[i] * H * d, w + (size_t)q_rows[i] * H,
                         k + (size_t)keys[i] * d, H, d);
}

/* ---------------------------------------------------------------------------
 * Top-k by full sort: score descending, then key index ascending.
 * ------------------------------------------------------------------------ */
typedef struct {
  double score;
  int64_t key;
} rec_t;

static int rec_cmp(const void *pa, const void *pb) {
  const rec_t *a = (const rec_t *)pa, *b = (const rec_t *)pb;
  if (a->score > b->score) return -1;
  if (a->score < b->score) return 1;
  return (a->key < b->key) ? -1 : (a->key > b->key);
}

/* Sorts recs[0..n) and writes the first min(topk, n) entries, padding the
 * rest of the row with (-1, -inf). */
static void emit_topk(rec_t *recs, int64_t n, int topk, int32_t *out_idx,
                      double *out_score) {
  qsort(recs, (size_t)n, sizeof(rec_t), rec_cmp);
  int64_t m = n < topk ? n : topk;
  for (int64_t i = 0; i < topk; ++i) {
    if (i < m) {
      out_idx[i] = (int32_t)recs[i].key;
      out_score[i] = recs[i].score;
    } else {
      out_idx[i] = -1;
      out_score[i] = -INFINITY;
    }
  }
}

/* ---------------------------------------------------------------------------
 * Chunked causal prefill: query row t (0 <= t < T_q) sits at position
 * p_t = q_offset + t and sees keys 0..p_t.  Only the rows listed in rows[]
 * are computed (all rows, or a sample).  For each listed row i:
 *   out_idx/out_score[i][0..topk)  the sorted Top-m (m = min(topk, p_t+1)),
 *   out_absmax[i]                  max_s |I(t,s)| over visible s,
 *   out_scores[i][0..T_k) (optional, may be NULL) every visible score, with
 *                                  -inf past p_t.
 * ------------------------------------------------------------------------ */
OR_API int oracle_prefill_topk(const uint16_t *q, const float *w, const uint16_t *k,
                               int64_t q_offset, int64_t T_q, int64_t T_k, int H, int d,
                               int topk, const int64_t *rows, int64_t n_rows,
                               int32_t *out_idx, double *out_score, double *out_absmax,
                               double *out_scores, int n_threads) {
  if (q_offset < 0 || q_offset + T_q > T_k || topk <= 0) return -1;
  for (int64_t i = 0; i < n_rows; ++i)
    if (rows[i] < 0 || rows[i] >= T_q) return -1;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int64_t i = 0; i < n_rows; ++i) {
    int64_t t = rows[i];
    int64_t nvis = q_offset + t + 1;
    const uint16_t *q_row = q + (size_t)t * H * d;
    const float *w_row = w + (size_t)t * H;
    rec_t *recs = (rec_t *)malloc(sizeof(rec_t) * (size_t)nvis);
    double amax = 0.0;
    for (int64_t s = 0; s < nvis; ++s) {
      double I = index_score(q_row, w_row, k + (size_t)s * d, H, d);
      recs[s].score = I;
      recs[s].key = s;
      if (fabs(I) > amax) amax = fabs(I);
      if (out_scores) out_scores[(size_t)i * T_k + s] = I;
    }
    if (out_scores)
      for (int64_t s = nvis; s < T_k; ++s) out_scores[(size_t)i * T_k + s] = -INFINITY;
    out_absmax[i] = amax;
    emit_topk(recs, nvis, topk, out_idx + (size_t)i * topk, out_score + (size_t)i * topk);
    free(recs);
  }
  return 0;
}

/* ---------------------------------------------------------------------------
 * Batched decode: sequence b has one query q[b] (H x d) and its own key cache
 * k[b] (t_cap x d) of which the first seq_len[b] keys are visible (the decode
 * scan over the whole cache, "DeepSeek DSA FLOPs", Decode).
 * ------------------------------------------------------------------------ */
OR_API int oracle_decode_topk(const uint16_t *q, const float *w, const uint16_t *k,
                              const int32_t *seq_len, int64_t B, int64_t t_cap, int H,
                              int d, int topk, int32_t *out_idx, double *out_score,
                              double *out_absmax, int n_threads) {
  if (topk <= 0) return -1;
  for (int64_t b = 0; b < B; ++b)
    if (seq_len[b] < 0 || seq_len[b] > t_cap) return -1;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int64_t b = 0; b < B; ++b) {
    int64_t n = seq_len[b];
    const uint16_t *kb = k + (size_t)b * t_cap * d;
    rec_t *recs = (rec_t *)malloc(sizeof(rec_t) * (size_t)(n > 0 ? n : 1));
    double amax = 0.0;
    for (int64_t s = 0; s < n; ++s) {
      double I = index_score(q + (size_t)b * H * d, w + (size_t)b * H, kb + (size_t)s * d, H, d);
      recs[s].score = I;
      recs[s].key = s;
      if (fabs(I) > amax) amax = fabs(I);
    }
    out_absmax[b] = amax;
    emit_topk(recs, n, topk, out_idx + (size_t)b * topk, out_score + (size_t)b * topk);
    free(recs);
  }
  return 0;
}

/* ---------------------------------------------------------------------------
 * DoSA certified pruning, in fp64 ("DoSA: Dots Sparse Attention", steps 1-3;
 * 163.com write-up, section 03).  This is the checker for the method's
 * mathematics: the plan, the per-key upper bound U(t,s), the seed threshold
 * tau_t, and the pruned selection, which must equal the dense selection.
 *
 * Plan for one query row (computed once, reused for every key):
 *  - importance_j = |w_j| * mean over the sampled seed keys of ReLU(q_j . k);
 *    the r heads of largest importance (ties: smaller j) are the retained set R.
 *  - omitted heads with w_j > 0 form P, with w_j < 0 form N (w_j = 0 heads
 *    contribute nothing and are dropped).
 *  - for j in P: c_j = least-squares coefficients of q_j on {q_i : i in R}
 *    (any coefficients keep the bound valid; least squares keeps it tight),
 *    residual r_j = q_j - sum_i c_ji q_i, rho_j = ||r_j||.
 *  - two auxiliary rows: q_pos = sum_P w_j q_j and q_neg = sum_N |w_j| q_j;
 *    alpha_i = sum_P w_j |c_ji|, beta = sum_P w_j rho_j.
 *
 * Bound, with d_i = q_i . k:
 *  positive omitted heads, using w ReLU(x) = (w x + w |x|) / 2 and
 *  |x_j| <= sum_i |c_ji| |d_i| + rho_j ||k||  (Cauchy-Schwarz on the residual):
 *      sum_P w_j ReLU(x_j) <= q_pos.k / 2 + (sum_R alpha_i |d_i| + beta ||k||) / 2
 *  negative omitted heads, sum-then-ReLU is a lower bound on their penalty:
 *      sum_N |w_j| ReLU(x_j) >= ReLU(q_neg . k)
 *  U = sum_R w_i ReLU(d_i) + q_pos.k/2 + (sum_R alpha_i|d_i| + beta||k||)/2
 *      - ReLU(q_neg . k)   >=   I(t,s).
 * A key is pruned iff U < tau (strictly).
 * ------------------------------------------------------------------------ */

/* Plan layout (doubles), for H heads of width d and r retained heads:
 *   [0]            r_eff (number of retained heads actually used)
 *   [1 .. 1+H)     role per head: 0 retained, 1 positive omitted, 2 negative
 *                  omitted, 3 zero weight
 *   [1+H .. 1+2H)  alpha per head (nonzero only for retained heads)
 *   [1+2H]         beta
 *   [2+2H .. 2+2H+d)      q_pos
 *   [2+2H+d .. 2+2H+2d)   q_neg
 * Size: 2 + 2H + 2d. */
#define PLAN_SIZE(H, d) (2 + 2 * (H) + 2 * (d))

static int cholesky_solve(int n, double *G, double *b) {
  /* In-place Cholesky of the n x n SPD matrix G (row-major); solves G x = b
   * into b.  Returns -1 if G is not numerically positive definite. */
  for (int j = 0; j < n; ++j) {
    double s = G[j * n + j];
    for (int p = 0; p < j; ++p) s -= G[j * n + p] * G[j * n + p];
    if (!(s > 1e-12 * (1.0 + fabs(G[j * n + j])))) return -1;
    double ljj = sqrt(s);
    G[j * n + j] = ljj;
    for (int i = j + 1; i < n; ++i) {
      double v = G[i * n + j];
      for (int p = 0; p < j; ++p) v -= G[i * n + p] * G[j * n + p];
      G[i * n + j] = v / ljj;
    }
  }
  for (int i = 0; i < n; ++i) {
    double v = b[i];
    for (int p = 0; p < i; ++p) v -= G[i * n + p] * b[p];
    b[i] = v / G[i * n + i];
  }
  for (int i = n - 1; i >= 0; --i) {
    double v = b[i];
    for (int p = i + 1; p < n; ++p) v -= G[p * n + i] * b[p];
    b[i] = v / G[i * n + i];
  }
  return 0;
}

OR_API int oracle_dosa_plan_size(int H, int d) { return PLAN_SIZE(H, d); }

OR_API int oracle_dosa_plan(const uint16_t *q_row, const float *w_row,
                            const uint16_t *k, const int32_t *sample_keys, int n_sample,
                            int H, int d, int r, double *plan) {
  if (r < 0 || r > H || H > 256 || d > 256) return -1;
  double *imp = (double *)calloc((size_t)H, sizeof(double));
  int *order = (int *)malloc(sizeof(int) * (size_t)H);
  for (int j = 0; j < H; ++j) {
    double acc = 0.0;
    for (int s = 0; s < n_sample; ++s) {
      double x = dot_f64(q_row + (size_t)j * d, k + (size_t)sample_keys[s] * d, d);
      acc += x > 0.0 ? x : 0.0;
    }
    imp[j] = fabs((double)w_row[j]) * (n_sample > 0 ? acc / n_sample : 0.0);
    order[j] = j;
  }
  /* stable selection of the r largest importances (ties: smaller j first) */
  for (int a = 0; a < H; ++a)
    for (int b = a + 1; b < H; ++b)
      if (imp[order[b]] > imp[order[a]] ||
          (imp[order[b]] == imp[order[a]] && order[b] < order[a])) {
        int tmp = order[a];
        order[a] = order[b];
        order[b] = tmp;
      }
  double *role = plan + 1, *alpha = plan + 1 + H, *beta = plan + 1 + 2 * H;
  double *qpos = plan + 2 + 2 * H, *qneg = plan + 2 + 2 * H + d;
  memset(plan, 0, sizeof(double) * (size_t)PLAN_SIZE(H, d));
  int R[256];
  for (int j = 0; j < H; ++j) role[j] = -1;
  for (int a = 0; a < r; ++a) {
    R[a] = order[a];
    role[order[a]] = 0;
  }
  plan[0] = r;
  for (int j = 0; j < H; ++j) {
    if (role[j] == 0) continue;
    role[j] = w_row[j] > 0.0f ? 1 : (w_row[j] < 0.0f ? 2 : 3);
  }
  /* Gram matrix of the retained rows */
  double *G = (double *)malloc(sizeof(double) * (size_t)(r * r + 1));
  double *Gw = (double *)malloc(sizeof(double) * (size_t)(r * r + 1));
  double *c = (double *)malloc(sizeof(double) * (size_t)(r + 1));
  double *qr = (double *)malloc(sizeof(double) * (size_t)d);
  for (int a = 0; a < r; ++a)
    for (int b = 0; b < r; ++b)
      G[a * r + b] = dot_f64(q_row + (size_t)R[a] * d, q_row + (size_t)R[b] * d, d);
  *beta = 0.0;
  for (int j = 0; j < H; ++j) {
    const uint16_t *qj = q_row + (size_t)j * d;
    double wj = (double)w_row[j];
    if (role[j] == 2) {
      for (int i = 0; i < d; ++i) qneg[i] += fabs(wj) * bf16_to_f64(qj[i]);
      continue;
    }
    if (role[j] != 1) continue;
    for (int i = 0; i < d; ++i) qpos[i] += wj * bf16_to_f64(qj[i]);
    /* least-squares coefficients; zeros if the Gram matrix is singular */
    for (int a = 0; a < r; ++a) c[a] = dot_f64(q_row + (size_t)R[a] * d, qj, d);
    memcpy(Gw, G, sizeof(double) * (size_t)(r * r));
    if (r == 0 || cholesky_solve(r, Gw, c) != 0)
      for (int a = 0; a < r; ++a) c[a] = 0.0;
    for (int i = 0; i < d; ++i) qr[i] = bf16_to_f64(qj[i]);
    for (int a = 0; a < r; ++a)
      for (int i = 0; i < d; ++i) qr[i] -= c[a] * bf16_to_f64(q_row[(size_t)R[a] * d + i]);
    double rho2 = 0.0;
    for (int i = 0; i < d; ++i) rho2 += qr[i] * qr[i];
    *beta += wj * sqrt(rho2);
    for (int a = 0; a < r; ++a) alpha[R[a]] += wj * fabs(c[a]);
  }
  free(G);
  free(Gw);
  free(c);
  free(qr);
  free(imp);
  free(order);
  return 0;
}

OR_API double oracle_dosa_bound(const double *plan, const uint16_t *q_row,
                                const float *w_row, const uint16_t *k_s, int H, int d) {
  const double *role = plan + 1, *alpha = plan + 1 + H;
  double beta = plan[1 + 2 * H];
  const double *qpos = plan + 2 + 2 * H, *qneg = plan + 2 + 2 * H + d;
  double U = 0.0, res = 0.0, kn2 = 0.0, dpos = 0.0, dneg = 0.0;
  for (int i = 0; i < d; ++i) {
    double kv = bf16_to_f64(k_s[i]);
    kn2 += kv * kv;
    dpos += qpos[i] * kv;
    dneg += qneg[i] * kv;
  }
  for (int j = 0; j < H; ++j) {
    if (role[j] != 0) continue;
    double x = dot_f64(q_row + (size_t)j * d, k_s, d);
    U += (double)w_row[j] * (x > 0.0 ? x : 0.0);
    res += alpha[j] * fabs(x);
  }
  U += 0.5 * dpos + 0.5 * (res + beta * sqrt(kn2)) - (dneg > 0.0 ? dneg : 0.0);
  return U;
}

/* Planner sample of the seed list ("DoSA" reading notes, annotation
 * ADQKPC5Q, step 1: 128 positions 32 + 64 i of the seed region).  Reading:
 * the midpoints of 128 equal slices of the first n' = min(n_seed, 8192) seed
 * entries, entry floor((2i+1) n' / (2m)) for i < m = min(128, n'); at
 * n' = 8192 these are exactly the positions 32 + 64 i, and shorter seed
 * lists keep the same even spacing. */
OR_API int oracle_dosa_sample(const int32_t *seeds, int n_seed, int32_t *out) {
  int n = n_seed < 8192 ? n_seed : 8192;
  int m = n < 128 ? n : 128;
  for (int i = 0; i < m; ++i) out[i] = seeds[((int64_t)(2 * i + 1) * n) / (2 * m)];
  return m;
}

/* The whole pruned selection for one row at position p (keys 0..p visible).
 * Seeds must be distinct, visible, and at least topk of them.
 * Outputs: out_idx/out_score (topk, sorted, padded), *tau, counters
 * stats[0] screened keys (non-seed visible), stats[1] survivors (U >= tau),
 * stats[2] records written (seed + refined scores >= tau),
 * and *min_gap = min over screened keys of U - I (>= 0 if the bound holds).
 * U_out (optional, length p+1) receives U for screened keys, NAN for seeds. */
OR_API int oracle_dosa_row(const uint16_t *q_row, const float *w_row, const uint16_t *k,
                           int64_t p, const int32_t *seeds, int n_seed, int topk, int r,
                           int H, int d, int32_t *out_idx, double *out_score, double *tau,
                           int64_t *stats, double *min_gap, double *U_out) {
  int64_t nvis = p + 1;
  if (n_seed < topk || topk <= 0) return -1;
  unsigned char *is_seed = (unsigned char *)calloc((size_t)nvis, 1);
  for (int i = 0; i < n_seed; ++i) {
    if (seeds[i] < 0 || seeds[i] > p || is_seed[seeds[i]]) {
      free(is_seed);
      return -4;
    }
    is_seed[seeds[i]] = 1;
  }
  /* step 1: seed scores with all heads; tau is the topk-th largest */
  rec_t *recs = (rec_t *)malloc(sizeof(rec_t) * (size_t)(nvis));
  for (int i = 0; i < n_seed; ++i) {
    recs[i].key = seeds[i];
    recs[i].score = index_score(q_row, w_row, k + (size_t)seeds[i] * d, H, d);
  }
  qsort(recs, (size_t)n_seed, sizeof(rec_t), rec_cmp);
  double t = recs[topk - 1].score;
  *tau = t;
  int64_t n_rec = 0;
  for (int i = 0; i < n_seed; ++i)
    if (recs[i].score >= t) recs[n_rec++] = recs[i];
  /* plan */
  int32_t sample[128];
  int m = oracle_dosa_sample(seeds, n_seed, sample);
  double *plan = (double *)malloc(sizeof(double) * (size_t)PLAN_SIZE(H, d));
  oracle_dosa_plan(q_row, w_row, k, sample, m, H, d, r, plan);
  /* step 2 (screen) and step 3 (refine, keep scores >= tau) */
  int64_t screened = 0, survivors = 0;
  double gap = INFINITY;
  for (int64_t s = 0; s < nvis; ++s) {
    if (is_seed[s]) {
      if (U_out) U_out[s] = NAN;
      continue;
    }
    ++screened;
    double U = oracle_dosa_bound(plan, q_row, w_row, k + (size_t)s * d, H, d);
    double I = index_score(q_row, w_row, k + (size_t)s * d, H, d);
    if (U_out) U_out[s] = U;
    if (U - I < gap) gap = U - I;
    if (U < t) continue; /* certified: cannot reach the Top-k */
    ++survivors;
    if (I >= t) {
      recs[n_rec].key = s;
      recs[n_rec].score = I;
      ++n_rec;
    }
  }
  stats[0] = screened;
  stats[1] = survivors;
  stats[2] = n_rec;
  *min_gap = gap;
  emit_topk(recs, n_rec, topk, out_idx, out_score);
  free(plan);
  free(recs);
  free(is_seed);
  return 0;
}

/* ---------------------------------------------------------------------------
 * FP8 indexer scoring ("DeepSeek DSA FLOPs", Lightning Indexer: the indexer
 * runs in FP8).  Reading: q and k are stored as FP8 E4M3 codes with one fp32
 * scale per stored row (per query head row and per key), so the real vectors
 * are q(t,j) = q_scale(t,j) * e4m3(q8(t,j)) and k(s) = k_scale(s) * e4m3(k8(s)),
 * and the index score is the same definition on them:
 *     I(t,s) = sum_j w(t,j) * ReLU(q(t,j) . k(s)).
 * ------------------------------------------------------------------------ */
/* OCP FP8 E4M3 ("FN"): sign, 4 exponent bits with bias 7, 3 mantissa bits;
 * exponent field 0 holds the subnormals m/8 * 2^-6; no infinities; the
 * all-ones exponent and mantissa pattern is NaN. */
static double e4m3_to_f64(uint8_t b) {
  int sgn = b >> 7, e = (b >> 3) & 15, m = b & 7;
  if (e == 15 && m == 7) return NAN;
  double v = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
  return sgn ? -v : v;
}

OR_API void oracle_e4m3_decode(const uint8_t *codes, int64_t n, double *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_to_f64(codes[i]);
}

/* The 256 code values, filled from e4m3_to_f64 by the (serial) entry points
 * before any parallel region reads it. */
static double g_e4m3[256];
static void e4m3_table(void) {
  for (int c = 0; c < 256; ++c) g_e4m3[c] = e4m3_to_f64((uint8_t)c);
}

static double index_score_fp8(const uint8_t *q_row, const float *qs_row, const float *w_row,
                              const uint8_t *k_s, double ks, int H, int d) {
  double I = 0.0;
  for (int j = 0; j < H; ++j) {
    double x = 0.0, qs = (double)qs_row[j];
    for (int i = 0; i < d; ++i) x += (qs * g_e4m3[q_row[(size_t)j * d + i]]) * (ks * g_e4m3[k_s[i]]);
    I += (double)w_row[j] * (x > 0.0 ? x : 0.0);
  }
  return I;
}

/* The FP8 chunked causal prefill: as oracle_prefill_topk, on FP8 inputs. */
OR_API int oracle_prefill_topk_fp8(const uint8_t *q, const float *q_scale, const float *w,
                                   const uint8_t *k, const float *k_scale, int64_t q_offset,
                                   int64_t T_q, int64_t T_k, int H, int d, int topk,
                                   const int64_t *rows, int64_t n_rows, int32_t *out_idx,
                                   double *out_score, double *out_absmax, int n_threads) {
  if (q_offset < 0 || q_offset + T_q > T_k || topk <= 0) return -1;
  for (int64_t i = 0; i < n_rows; ++i)
    if (rows[i] < 0 || rows[i] >= T_q) return -1;
  e4m3_table();
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int64_t i = 0; i < n_rows; ++i) {
    int64_t t = rows[i];
    int64_t nvis = q_offset + t + 1;
    rec_t *recs = (rec_t *)malloc(sizeof(rec_t) * (size_t)nvis);
    double amax = 0.0;
    for (int64_t s = 0; s < nvis; ++s) {
      double I = index_score_fp8(q + (size_t)t * H * d, q_scale + (size_t)t * H, w + (size_t)t * H,
                                 k + (size_t)s * d, (double)k_scale[s], H, d);
      recs[s].score = I;
      recs[s].key = s;
      if (fabs(I) > amax) amax = fabs(I);
    }
    out_absmax[i] = amax;
    emit_topk(recs, nvis, topk, out_idx + (size_t)i * topk, out_score + (size_t)i * topk);
    free(recs);
  }
  return 0;
}

/* Scores of arbitrary (query row, key) pairs of FP8 inputs. */
OR_API void oracle_score_pairs_fp8(const uint8_t *q, const float *q_scale, const float *w,
                                   const uint8_t *k, const float *k_scale, int H, int d, int64_t n,
                                   const int64_t *q_rows, const int64_t *keys, double *out,
                                   int n_threads) {
  e4m3_table();
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 64)
#endif
  for (int64_t i = 0; i < n; ++i)
    out[i] = index_score_fp8(q + (size_t)q_rows[i] * H * d, q_scale + (size_t)q_rows[i] * H,
                             w + (size_t)q_rows[i] * H, k + (size_t)keys[i] * d,
                             (double)k_scale[keys[i]], H, d);
}

/* ---------------------------------------------------------------------------
 * Seeds from historical selection frequency (163.com write-up, section 03:
 * seed candidates may be chosen by how often keys were selected before).
 * Reading: count, over earlier query rows' Top-k lists prev[n_rows][topk]
 * (-1 padding ignored), how many rows selected each key s < n_keys; the seeds
 * are the n_seed keys with the largest counts, ties broken by the smaller
 * key (keys never selected fill up from key 0), listed in ascending key order.
 * ------------------------------------------------------------------------ */
typedef struct {
  int64_t count;
  int64_t key;
} freq_t;

static int freq_cmp(const void *pa, const void *pb) {
  const freq_t *a = (const freq_t *)pa, *b = (const freq_t *)pb;
  if (a->count != b->count) return a->count > b->count ? -1 : 1;
  return (a->key < b->key) ? -1 : (a->key > b->key);
}

OR_API int oracle_seeds_from_history(const int32_t *prev, int64_t n_rows, int topk, int64_t n_keys,
                                     int n_seed, int32_t *seeds, int64_t *counts_out) {
  if (n_seed < 1 || n_seed > n_keys) return -1;
  freq_t *f = (freq_t *)malloc(sizeof(freq_t) * (size_t)n_keys);
  for (int64_t s = 0; s < n_keys; ++s) {
    f[s].count = 0;
    f[s].key = s;
  }
  for (int64_t i = 0; i < n_rows * topk; ++i)
    if (prev[i] >= 0 && prev[i] < n_keys) f[prev[i]].count += 1;
  if (counts_out)
    for (int64_t s = 0; s < n_keys; ++s) counts_out[s] = f[s].count;
  qsort(f, (size_t)n_keys, sizeof(freq_t), freq_cmp);
  unsigned char *pick = (unsigned char *)calloc((size_t)n_keys, 1);
  for (int i = 0; i < n_seed; ++i) pick[f[i].key] = 1;
  int n = 0;
  for (int64_t s = 0; s < n_keys; ++s)
    if (pick[s]) seeds[n++] = (int32_t)s;
  free(pick);
  free(f);
  return 0;
}

/* Pair counts and FLOP counts ("DeepSeek DSA FLOPs": causal pair count,
 * selected pair count, full-prefix scoring and decode FLOPs). */
OR_API double oracle_n_dense(double T) { return T * (T + 1.0) / 2.0; }

OR_API double oracle_n_sel(double T, double k) {
  double s = 0.0;
  for (double i = 1.0; i <= T; i += 1.0) s += (i < k ? i : k);
  return s;
}

/* Matrix-multiply FLOPs of index scoring over a set of visible pairs:
 * each pair costs one d-wide dot per head, i.e. 2*H*d FLOPs. */
OR_API double oracle_scoring_flops(double pairs, int H, int d) { return 2.0 * H * d * pairs; }
