/*
 * haste_ref.c -- plain, slow, fp64 CPU oracle of the HASTE group-shared fixed
 * fan-in output layer.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and
 * the CPU-baseline leg of the benchmark call it; the product path never does.
 * It shares no code, header or table with the CUDA library.
 *
 * Source: "HASTE: Hardware-Aware Dynamic Sparse Training for Large Output Spaces"
 * (summary page), Methodology 1 "Group-Shared Fixed Fan-In Sparsity":
 *   - Structure: labels are partitioned into groups; every label of a group uses
 *     the same sparse set of input-feature indices (the fan-in pattern) but keeps
 *     its own weight vector.
 *   - Memory efficiency: indices are stored once per group, not once per label.
 * Methodology 2 "Head-Tail Decomposition": a dense classifier for the frequent
 * head labels (computed by the numpy part of the oracle, oracle.py).
 *
 * Readings where the page is silent (each also listed in the design notes):
 *   - groups are contiguous label ranges: group g owns labels [g*G, g*G+G);
 *   - group g's index set idx[g, 0..k) is strictly increasing in [0, d);
 *   - W is [L, k]: W[l, s] multiplies feature idx[l / G, s];
 *   - the loss is binary cross-entropy with logits against sparse positive lists,
 *     summed over labels and scaled by `scale` (1/B: mean over the batch).
 *
 * Each array carries its own type code: fp32 (0), bf16 bit patterns (1) or
 * double (2); all widen exactly to double.  All sums run in double in the order written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define REF_OK 0
#define REF_ERR_ARG 1
#define REF_ERR_UNSORTED 2
#define REF_ERR_RANGE 3

static inline double ld(const void* p, int64_t i, int dt) {
  if (dt == 0) return (double)((const float*)p)[i];
  if (dt == 2) return ((const double*)p)[i];
  uint32_t u = ((uint32_t)((const uint16_t*)p)[i]) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Validation of the fan-in sets: the first offending element in row-major order
 * decides the status (out of range before ordering). */
int ref_validate(const int32_t* idx, int64_t n_groups, int32_t k, int32_t d) {
  if (!idx || n_groups <= 0 || k <= 0 || d <= 0) return REF_ERR_ARG;
  for (int64_t g = 0; g < n_groups; ++g) {
    const int32_t* row = idx + g * (int64_t)k;
    for (int32_t s = 0; s < k; ++s) {
      if (row[s] < 0 || row[s] >= d) return REF_ERR_RANGE;
      if (s > 0 && row[s] <= row[s - 1]) return REF_ERR_UNSORTED;
    }
  }
  return REF_OK;
}

/* Inverse map feature -> (group, slot).  inv_off[f] = number of entries whose
 * feature is below f; the entries e = g*k + s of feature f follow in ascending g
 * (a stable counting sort of the entries by feature). */
int ref_plan(const int32_t* idx, int64_t n_groups, int32_t k, int32_t d,
             int32_t* inv_off, int32_t* inv_ent) {
  int st = ref_validate(idx, n_groups, k, d);
  if (st != REF_OK) return st;
  int64_t n = n_groups * (int64_t)k;
  int64_t* cnt = (int64_t*)calloc((size_t)d + 1, sizeof(int64_t));
  if (!cnt) return REF_ERR_ARG;
  for (int64_t e = 0; e < n; ++e) cnt[idx[e] + 1] += 1;
  for (int32_t f = 0; f < d; ++f) cnt[f + 1] += cnt[f];
  for (int32_t f = 0; f <= d; ++f) inv_off[f] = (int32_t)cnt[f];
  for (int64_t g = 0; g < n_groups; ++g)
    for (int32_t s = 0; s < k; ++s) {
      int32_t f = idx[g * k + s];
      inv_ent[cnt[f]++] = (int32_t)(g * k + s);
    }
  free(cnt);
  return REF_OK;
}

/* Forward: logits[b, g*G+j] = sum_{s<k} X[b, idx[g,s]] * W[g*G+j, s]. */
void ref_forward(int dx_, const void* X, int dw_, const void* W, const int32_t* idx, int32_t B,
                 int32_t d, int64_t n_groups, int32_t G, int32_t k, double* logits) {
  int64_t L = n_groups * G;
#pragma omp parallel for schedule(static)
  for (int32_t b = 0; b < B; ++b)
    for (int64_t g = 0; g < n_groups; ++g)
      for (int32_t j = 0; j < G; ++j) {
        int64_t l = g * G + j;
        double acc = 0.0;
        for (int32_t s = 0; s < k; ++s)
          acc += ld(X, (int64_t)b * d + idx[g * k + s], dx_) * ld(W, l * k + s, dw_);
        logits[(int64_t)b * L + l] = acc;
      }
}

/* dW[g*G+j, s] = sum_{b<B} dY[b, g*G+j] * X[b, idx[g,s]]. */
void ref_backward_dw(int dx_, const void* X, int dy_, const void* dY, const int32_t* idx, int32_t B,
                     int32_t d, int64_t n_groups, int32_t G, int32_t k, double* dW) {
  int64_t L = n_groups * G;
#pragma omp parallel for schedule(static)
  for (int64_t g = 0; g < n_groups; ++g)
    for (int32_t j = 0; j < G; ++j)
      for (int32_t s = 0; s < k; ++s) {
        int64_t l = g * G + j;
        double acc = 0.0;
        for (int32_t b = 0; b < B; ++b)
          acc += ld(dY, (int64_t)b * L + l, dy_) * ld(X, (int64_t)b * d + idx[g * k + s], dx_);
        dW[l * k + s] = acc;
      }
}

/* dX[b, f] = sum_g sum_s [idx[g,s] == f] sum_j dY[b, g*G+j] * W[g*G+j, s];
 * groups in ascending order, features in no group stay exactly 0. */
void ref_backward_dx(int dw_, const void* W, int dy_, const void* dY, const int32_t* idx, int32_t B,
                     int32_t d, int64_t n_groups, int32_t G, int32_t k, double* dX) {
  int64_t L = n_groups * G;
#pragma omp parallel for schedule(static)
  for (int32_t b = 0; b < B; ++b) {
    double* row = dX + (int64_t)b * d;
    for (int32_t f = 0; f < d; ++f) row[f] = 0.0;
    for (int64_t g = 0; g < n_groups; ++g)
      for (int32_t s = 0; s < k; ++s) {
        double z = 0.0;
        for (int32_t j = 0; j < G; ++j) {
          int64_t l = g * G + j;
          z += ld(dY, (int64_t)b * L + l, dy_) * ld(W, l * k + s, dw_);
        }
        row[idx[g * k + s]] += z;
      }
  }
}

/* Binary cross-entropy with logits against sparse positives.
 * y[b,l] = 1 iff l is in row b of the CSR (row_ptr, ids); duplicates count once.
 * loss = scale * sum_{b,l} ( max(z,0) - z*y + log1p(exp(-|z|)) )
 * dY[b,l] = scale * (sigmoid(z) - y).  Returns the loss. */
static inline double sigmoid(double z) {
  if (z >= 0) return 1.0 / (1.0 + exp(-z));
  double e = exp(z);
  return e / (1.0 + e);
}

static inline int is_positive(const int32_t* ids, int32_t lo, int32_t hi, int64_t l) {
  for (int32_t i = lo; i < hi; ++i)
    if (ids[i] == l) return 1;
  return 0;
}

double ref_bce(const double* logits, const int32_t* row_ptr, const int32_t* ids, int32_t B,
               int64_t L, double scale, double* dY) {
  double* part = (double*)calloc((size_t)B, sizeof(double));
#pragma omp parallel for schedule(static)
  for (int32_t b = 0; b < B; ++b) {
    double acc = 0.0;
    for (int64_t l = 0; l < L; ++l) {
      double z = logits[(int64_t)b * L + l];
      double y = is_positive(ids, row_ptr[b], row_ptr[b + 1], l) ? 1.0 : 0.0;
      acc += (z > 0 ? z : 0.0) - z * y + log1p(exp(-fabs(z)));
      if (dY) dY[(int64_t)b * L + l] = scale * (sigmoid(z) - y);
    }
    part[b] = acc;
  }
  double loss = 0.0;
  for (int32_t b = 0; b < B; ++b) loss += part[b];
  free(part);
  return scale * loss;
}

/* ---- single-output evaluations for full-size sampled checks ---------------- */

static double logit_at(int dt, const void* X, const void* W, const int32_t* idx, int32_t d,
                       int32_t G, int32_t k, int32_t b, int64_t l) {
  int64_t g = l / G;
  double acc = 0.0;
  for (int32_t s = 0; s < k; ++s)
    acc += ld(X, (int64_t)b * d + idx[g * k + s], dt) * ld(W, l * k + s, dt);
  return acc;
}

/* logits at n sampled (b, l) pairs */
void ref_logits_at(int dt, const void* X, const void* W, const int32_t* idx, int32_t d,
                   int32_t G, int32_t k, int64_t n, const int32_t* bs, const int64_t* ls,
                   double* out) {
#pragma omp parallel for schedule(dynamic)
  for (int64_t i = 0; i < n; ++i) out[i] = logit_at(dt, X, W, idx, d, G, k, bs[i], ls[i]);
}

/* dY entry of the fused step: scale * (sigmoid(z) - y) with z recomputed. */
static double dy_fused_at(int dt, const void* X, const void* W, const int32_t* idx, int32_t d,
                          int32_t G, int32_t k, const int32_t* row_ptr, const int32_t* ids,
                          double scale, int32_t b, int64_t l) {
  double z = logit_at(dt, X, W, idx, d, G, k, b, l);
  double y = is_positive(ids, row_ptr[b], row_ptr[b + 1], l) ? 1.0 : 0.0;
  return scale * (sigmoid(z) - y);
}

/* dW at n sampled (l, s) pairs.  fused != 0: dY from the BCE step (row_ptr, ids,
 * scale); fused == 0: dY given as a [B, L] tensor of dtype dt. */
void ref_dw_at(int dt, const void* X, const void* W, const void* dY, const int32_t* idx,
               int32_t B, int32_t d, int64_t L, int32_t G, int32_t k, int fused,
               const int32_t* row_ptr, const int32_t* ids, double scale, int64_t n,
               const int64_t* ls, const int32_t* ss, double* out) {
#pragma omp parallel for schedule(dynamic)
  for (int64_t i = 0; i < n; ++i) {
    int64_t l = ls[i];
    int64_t g = l / G;
    int32_t f = idx[g * k + ss[i]];
    double acc = 0.0;
    for (int32_t b = 0; b < B; ++b) {
      double dy = fused ? dy_fused_at(dt, X, W, idx, d, G, k, row_ptr, ids, scale, b, l)
                        : ld(dY, (int64_t)b * L + l, dt);
      acc += dy * ld(X, (int64_t)b * d + f, dt);
    }
    out[i] = acc;
  }
}

/* dX at n sampled (b, f) pairs, summing over the groups that contain f (found by
 * scanning each group's index set), groups ascending. */
void ref_dx_at(int dt, const void* X, const void* W, const void* dY, const int32_t* idx,
               int32_t B, int32_t d, int64_t L, int32_t G, int32_t k, int fused,
               const int32_t* row_ptr, const int32_t* ids, double scale, int64_t n,
               const int32_t* bs, const int32_t* fs, double* out) {
  int64_t n_groups = L / G;
  (void)B;
#pragma omp parallel for schedule(dynamic)
  for (int64_t i = 0; i < n; ++i) {
    int32_t b = bs[i], f = fs[i];
    double acc = 0.0;
    for (int64_t g = 0; g < n_groups; ++g) {
      const int32_t* row = idx + g * k;
      for (int32_t s = 0; s < k; ++s) {
        if (row[s] != f) continue;
        for (int32_t j = 0; j < G; ++j) {
          int64_t l = g * G + j;
          double dy = fused ? dy_fused_at(dt, X, W, idx, d, G, k, row_ptr, ids, scale, b, l)
                            : ld(dY, (int64_t)b * L + l, dt);
          acc += dy * ld(W, l * k + s, dt);
        }
      }
    }
    out[i] = acc;
  }
}

/* ---- two-stage top-k scoring ------------------------------------------------
 * Source: "A Faster Generalized Two-Stage Approximate Top-K" (summary page),
 * Methodology: stage 1 splits the N scores into buckets and keeps the top K' of
 * each bucket; stage 2 returns the top K of the buckets' K' survivors (K' = K:
 * the exact top K).  Here the scores of one sample are the logits of its L tail
 * labels, and bucket j holds the labels of groups [j*n_g/nb, (j+1)*n_g/nb):
 * contiguous whole groups (this project's reading; the page analyses random
 * partitions).  Order: larger score first, equal scores by smaller label id.
 * For each requested sample row rows[i]: out_val[i*K + j], out_id[i*K + j]. */
static int ranks_before(double v1, int64_t i1, double v2, int64_t i2) {
  return v1 > v2 || (v1 == v2 && i1 < i2);
}
/* insert (v, id) into the list (vals, ids) of length n, kept in rank order */
static void keep_best(double* vals, int64_t* ids, int32_t n, double v, int64_t id) {
  if (!ranks_before(v, id, vals[n - 1], ids[n - 1])) return;
  int32_t j = n - 1;
  while (j > 0 && ranks_before(v, id, vals[j - 1], ids[j - 1])) {
    vals[j] = vals[j - 1];
    ids[j] = ids[j - 1];
    --j;
  }
  vals[j] = v;
  ids[j] = id;
}
void ref_topk(int dt, const void* X, const void* W, const int32_t* idx, int32_t d, int64_t n_groups,
              int32_t G, int32_t k, int32_t K, int32_t Kp, int32_t nb, int64_t n_rows, const int32_t* rows,
              double* out_val, int64_t* out_id) {
#pragma omp parallel for schedule(dynamic)
  for (int64_t i = 0; i < n_rows; ++i) {
    const int32_t b = rows[i];
    double* cv = (double*)malloc(sizeof(double) * (size_t)nb * Kp);
    int64_t* ci = (int64_t*)malloc(sizeof(int64_t) * (size_t)nb * Kp);
    for (int32_t j = 0; j < nb; ++j) {           /* stage 1: top Kp of bucket j */
      double* bv = cv + (size_t)j * Kp;
      int64_t* bi = ci + (size_t)j * Kp;
      for (int32_t e = 0; e < Kp; ++e) {
        bv[e] = -INFINITY;
        bi[e] = INT64_MAX;
      }
      const int64_t ga = (int64_t)j * n_groups / nb, gb = (int64_t)(j + 1) * n_groups / nb;
      for (int64_t l = ga * G; l < gb * G; ++l) keep_best(bv, bi, Kp, logit_at(dt, X, W, idx, d, G, k, b, l), l);
    }
    double* ov = out_val + i * K;                  /* stage 2: top K of the survivors */
    int64_t* oi = out_id + i * K;
    for (int32_t e = 0; e < K; ++e) {
      ov[e] = -INFINITY;
      oi[e] = INT64_MAX;
    }
    for (int64_t c = 0; c < (int64_t)nb * Kp; ++c) keep_best(ov, oi, K, cv[c], ci[c]);
    free(cv);
    free(ci);
  }
}

/* ---- the tail loss alone, for full-size checks ------------------------------
 * loss = scale * sum_{b,l} ( max(z,0) - z*y + log1p(exp(-|z|)) ) with
 * z[b, l] = logits of the forward above, computed group by group without storing
 * the B x L logits: per group, the gathered inputs X[b, idx[g, s]] and the G
 * weight rows are widened once, then every logit is the sum over s ascending.
 * Per-group partial sums are added in group order (the result does not depend on
 * the thread count). */
double ref_bce_loss(int dt, const void* X, const void* W, const int32_t* idx, int32_t B, int32_t d,
                    int64_t n_groups, int32_t G, int32_t k, const int32_t* row_ptr, const int32_t* ids,
                    double scale) {
  double* part = (double*)calloc((size_t)n_groups, sizeof(double));
  if (!part) return NAN;
#pragma omp parallel
  {
    double* xg = (double*)malloc(sizeof(double) * (size_t)B * k);
    double* wg = (double*)malloc(sizeof(double) * (size_t)G * k);
#pragma omp for schedule(static)
    for (int64_t g = 0; g < n_groups; ++g) {
      for (int32_t b = 0; b < B; ++b)
        for (int32_t s = 0; s < k; ++s) xg[(int64_t)b * k + s] = ld(X, (int64_t)b * d + idx[g * k + s], dt);
      for (int32_t j = 0; j < G; ++j)
        for (int32_t s = 0; s < k; ++s) wg[(int64_t)j * k + s] = ld(W, (g * G + j) * k + s, dt);
      double acc = 0.0;
      for (int32_t b = 0; b < B; ++b)
        for (int32_t j = 0; j < G; ++j) {
          const int64_t l = g * G + j;
          double z = 0.0;
          for (int32_t s = 0; s < k; ++s) z += xg[(int64_t)b * k + s] * wg[(int64_t)j * k + s];
          const double y = is_positive(ids, row_ptr[b], row_ptr[b + 1], l) ? 1.0 : 0.0;
          acc += (z > 0 ? z : 0.0) - z * y + log1p(exp(-fabs(z)));
        }
      part[g] = acc;
    }
    free(xg);
    free(wg);
  }
  double loss = 0.0;
  for (int64_t g = 0; g < n_groups; ++g) loss += part[g];
  free(part);
  return scale * loss;
}
