/*
 * oracle.c -- plain, slow CPU oracle for decode-time token-level sparse
 * attention with shared routing.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: it exists so that the tests, the package smoke check and
 * the CPU-baseline leg of the benchmark can check the CUDA library against an
 * independent, obviously correct implementation.  It shares no code, header,
 * table or constant with the CUDA sources.
 *
 * Sources (page title, section):
 *  [CLSA-bg]   "CLSAとは？ルーティング共有で128Kコンテキスト推論を17倍高速化する
 *              スパースアテンション", section 研究の背景と課題: sparse attention
 *              computes attention over a chosen subset of the cached tokens;
 *              token-level selection keeps the k highest-scoring tokens.
 *  [CLSA-mech] same page, section CLSAの仕組み: one top-k index set per query
 *              token is computed once, over the one shared KV cache, and every
 *              cross-decoder layer reuses it unchanged.
 *  [Louver-pd] "技術サマリー：スパースアテンションを範囲検索問題として捉える",
 *              section 問題定義: keep every token whose score is above a
 *              threshold tau instead of a fixed count.
 *  [Louver-hs] same page, section 1. 半空間範囲検索への帰着: the kept set is
 *              the halfspace {p : <q,p> >= tau}; no key with score >= tau may
 *              be missed.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - score of key j for KV head h: the GQA group sum
 *        S = (sum_{g<G} sum_{i<d} q[h*G+g][i] * K[h][j][i]) * (1/sqrt(d)),
 *    query head hq belongs to KV head hq / G (contiguous groups);
 *  - scores are fp32 with the summation order written below (i ascending
 *    inside a head, then g ascending), each product and sum rounded to fp32
 *    (build with -ffp-contract=off so no fused multiply-add is formed);
 *    a double-precision variant exists to arbitrate boundary cases;
 *  - top-k ties at the k-th score go to the lower key index; -0.0 == +0.0;
 *  - threshold inclusion is inclusive (score >= tau), tau in score units;
 *  - index sets are returned in ascending key order;
 *  - attention is evaluated in double precision over the selected set; an
 *    empty set gives o = 0 and lse = -inf.
 *
 * Layouts (all dense, row-major): q [B,Hq,d]; K,V [B,Hkv,N,d]; S [B,Hkv,N];
 * idx [B,Hkv,stride]; count [B,Hkv]; per-layer queries [L,B,Hq,d];
 * out [L,B,Hq,d]; lse [L,B,Hq].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NONFINITE 2
#define ORACLE_NOMEM 3

static int shape_ok(int B, int N, int Hq, int Hkv, int d) {
  return B >= 1 && N >= 1 && Hq >= 1 && Hkv >= 1 && d >= 1 && Hq % Hkv == 0;
}

/* Routing scores in fp32 [CLSA-bg, CLSA-mech]. */
int oracle_scores_f32(int B, int N, int Hq, int Hkv, int d, const float *q,
                      const float *K, float *S) {
  if (!shape_ok(B, N, Hq, Hkv, d)) return ORACLE_BAD_ARG;
  const int G = Hq / Hkv;
  const float scale = (float)(1.0 / sqrt((double)d));
  int status = ORACLE_OK;
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hkv; ++h) {
      const float *Kh = K + ((size_t)b * Hkv + h) * (size_t)N * d;
      float *Sh = S + ((size_t)b * Hkv + h) * (size_t)N;
      for (int j = 0; j < N; ++j) {
        const float *kj = Kh + (size_t)j * d;
        float acc = 0.0f;
        for (int g = 0; g < G; ++g) {
          const float *qg = q + ((size_t)b * Hq + (size_t)h * G + g) * d;
          float part = 0.0f;
          for (int i = 0; i < d; ++i) {
            float prod = qg[i] * kj[i];
            part = part + prod;
          }
          acc = acc + part;
        }
        float s = acc * scale;
        if (!isfinite(s)) status = ORACLE_NONFINITE;
        Sh[j] = s;
      }
    }
  return status;
}

/* The same scores in double precision, used to arbitrate keys whose fp32
 * score sits on the selection boundary. */
int oracle_scores_f64(int B, int N, int Hq, int Hkv, int d, const float *q,
                      const float *K, double *S) {
  if (!shape_ok(B, N, Hq, Hkv, d)) return ORACLE_BAD_ARG;
  const int G = Hq / Hkv;
  const double scale = 1.0 / sqrt((double)d);
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hkv; ++h) {
      const float *Kh = K + ((size_t)b * Hkv + h) * (size_t)N * d;
      double *Sh = S + ((size_t)b * Hkv + h) * (size_t)N;
      for (int j = 0; j < N; ++j) {
        const float *kj = Kh + (size_t)j * d;
        double acc = 0.0;
        for (int g = 0; g < G; ++g) {
          const float *qg = q + ((size_t)b * Hq + (size_t)h * G + g) * d;
          for (int i = 0; i < d; ++i) acc += (double)qg[i] * (double)kj[i];
        }
        Sh[j] = acc * scale;
      }
    }
  return ORACLE_OK;
}

typedef struct {
  float s;
  int j;
} scored_t;

/* Descending score, then ascending index.  Float comparison treats -0.0 and
 * +0.0 as equal, which is the intended tie rule. */
static int by_score_desc_index_asc(const void *a, const void *b) {
  const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->j > y->j) - (x->j < y->j);
}

static int by_int_asc(const void *a, const void *b) {
  int x = *(const int *)a, y = *(const int *)b;
  return (x > y) - (x < y);
}

/* Top-k per row of S [BH, N]: the k highest scores, ties to the lower index,
 * written ascending into idx [BH, k] [CLSA-bg: "the k highest-scoring
 * tokens"; CLSA-mech: one set per query token]. */
int oracle_topk(int BH, int N, const float *S, int k, int *idx) {
  if (BH < 1 || N < 1 || k < 1 || k > N) return ORACLE_BAD_ARG;
  for (size_t t = 0; t < (size_t)BH * N; ++t)
    if (!isfinite(S[t])) return ORACLE_NONFINITE;
  int status = ORACLE_OK;
#pragma omp parallel for schedule(static)
  for (int r = 0; r < BH; ++r) {
    scored_t *all = (scored_t *)malloc((size_t)N * sizeof(scored_t));
    if (!all) {
      status = ORACLE_NOMEM;
      continue;
    }
    for (int j = 0; j < N; ++j) {
      all[j].s = S[(size_t)r * N + j];
      all[j].j = j;
    }
    qsort(all, (size_t)N, sizeof(scored_t), by_score_desc_index_asc);
    int *out = idx + (size_t)r * k;
    for (int t = 0; t < k; ++t) out[t] = all[t].j;
    qsort(out, (size_t)k, sizeof(int), by_int_asc);
    free(all);
  }
  return status;
}

/* Threshold set per row: every j with S >= tau[row], ascending
 * [Louver-pd, Louver-hs].  count[row] is the true size of the set; only the
 * first min(count, cap) indices (the lowest ones) are written. */
int oracle_threshold(int BH, int N, const float *S, const float *tau, int cap,
                     int *idx, int *count) {
  if (BH < 1 || N < 1 || cap < 1) return ORACLE_BAD_ARG;
  for (int r = 0; r < BH; ++r) {
    if (!isfinite(tau[r])) return ORACLE_NONFINITE;
    int c = 0;
    for (int j = 0; j < N; ++j) {
      float s = S[(size_t)r * N + j];
      if (!isfinite(s)) return ORACLE_NONFINITE;
      if (s >= tau[r]) {
        if (c < cap) idx[(size_t)r * cap + c] = j;
        ++c;
      }
    }
    count[r] = c;
  }
  return ORACLE_OK;
}

/* Nearest-rank p-th percentile per row, p = num/den: tau = the
 * ceil(p*N)-th smallest score.  Workload recipe for the threshold variant
 * (tau per head at a fixed percentile); not part of the method itself. */
static int by_float_asc(const void *a, const void *b) {
  float x = *(const float *)a, y = *(const float *)b;
  return (x > y) - (x < y);
}

int oracle_percentile_tau(int BH, int N, const float *S, int num, int den,
                          float *tau) {
  if (BH < 1 || N < 1 || num < 0 || den < 1 || num > den) return ORACLE_BAD_ARG;
  long long rank = ((long long)num * N + den - 1) / den; /* ceil(p*N) */
  if (rank < 1) rank = 1;
  float *row = (float *)malloc((size_t)N * sizeof(float));
  if (!row) return ORACLE_NOMEM;
  for (int r = 0; r < BH; ++r) {
    memcpy(row, S + (size_t)r * N, (size_t)N * sizeof(float));
    qsort(row, (size_t)N, sizeof(float), by_float_asc);
    tau[r] = row[rank - 1];
  }
  free(row);
  return ORACLE_OK;
}

/* Attention of every query head over the selected rows of its KV head
 * [CLSA-bg: attention over the selected subset; CLSA-mech: the same index
 * set for every layer].  Evaluated in double precision:
 *   z_j = <q, K_j> / sqrt(d),  m = max z,  w_j = exp(z_j - m),
 *   Z = sum w,  o = sum (w_j / Z) V_j,  lse = m + log Z.
 * q [Lq,B,Hq,d]; idx [B,Hkv,stride]; count [B,Hkv] or NULL (all = stride);
 * out [Lq,B,Hq,d] and lse [Lq,B,Hq] in double. */
int oracle_attn(int Lq, int B, int Hq, int Hkv, int d, int N, const float *q,
                const float *K, const float *V, const int *idx, int stride,
                const int *count, double *out, double *lse) {
  if (Lq < 1 || !shape_ok(B, N, Hq, Hkv, d) || stride < 1) return ORACLE_BAD_ARG;
  const int G = Hq / Hkv;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hkv; ++h) {
      int c = count ? count[b * Hkv + h] : stride;
      if (c < 0 || c > stride) return ORACLE_BAD_ARG;
      for (int t = 0; t < c; ++t) {
        int j = idx[((size_t)b * Hkv + h) * stride + t];
        if (j < 0 || j >= N) return ORACLE_BAD_ARG;
      }
    }
  const double scale = 1.0 / sqrt((double)d);
  int status = ORACLE_OK;
#pragma omp parallel for collapse(3) schedule(static)
  for (int l = 0; l < Lq; ++l)
    for (int b = 0; b < B; ++b)
      for (int hq = 0; hq < Hq; ++hq) {
        const int h = hq / G;
        const int c = count ? count[b * Hkv + h] : stride;
        const int *sel = idx + ((size_t)b * Hkv + h) * stride;
        const float *qv = q + (((size_t)l * B + b) * Hq + hq) * d;
        const float *Kh = K + ((size_t)b * Hkv + h) * (size_t)N * d;
        const float *Vh = V + ((size_t)b * Hkv + h) * (size_t)N * d;
        double *o = out + (((size_t)l * B + b) * Hq + hq) * d;
        double *ls = lse + ((size_t)l * B + b) * Hq + hq;
        for (int i = 0; i < d; ++i) o[i] = 0.0;
        if (c == 0) {
          *ls = -INFINITY;
          continue;
        }
        double *z = (double *)malloc((size_t)c * sizeof(double));
        if (!z) {
          status = ORACLE_NOMEM;
          continue;
        }
        double m = -INFINITY;
        for (int t = 0; t < c; ++t) {
          const float *kj = Kh + (size_t)sel[t] * d;
          double acc = 0.0;
          for (int i = 0; i < d; ++i) acc += (double)qv[i] * (double)kj[i];
          z[t] = acc * scale;
          if (z[t] > m) m = z[t];
        }
        double Z = 0.0;
        for (int t = 0; t < c; ++t) {
          z[t] = exp(z[t] - m);
          Z += z[t];
        }
        for (int t = 0; t < c; ++t) {
          const float *vj = Vh + (size_t)sel[t] * d;
          double w = z[t] / Z;
          for (int i = 0; i < d; ++i) o[i] += w * (double)vj[i];
        }
        *ls = m + log(Z);
        free(z);
      }
  return status;
}

/* One decode step: route once, then every layer attends over that one set
 * [CLSA-mech].  k > 0 selects the top-k mode; otherwise tau (per row) selects
 * the threshold mode with capacity cap and count written to count.  S is a
 * caller-provided [B,Hkv,N] fp32 scratch that receives the scores. */
int oracle_decode_step(int L, int B, int Hq, int Hkv, int d, int N,
                       const float *q_route, const float *q_layers,
                       const float *K, const float *V, int k, const float *tau,
                       int cap, float *S, int *idx, int *count, double *out,
                       double *lse) {
  int st = oracle_scores_f32(B, N, Hq, Hkv, d, q_route, K, S);
  if (st != ORACLE_OK) return st;
  int stride;
  if (k > 0) {
    st = oracle_topk(B * Hkv, N, S, k, idx);
    stride = k;
    if (st != ORACLE_OK) return st;
    return oracle_attn(L, B, Hq, Hkv, d, N, q_layers, K, V, idx, stride, NULL,
                       out, lse);
  }
  if (!tau) return ORACLE_BAD_ARG;
  st = oracle_threshold(B * Hkv, N, S, tau, cap, idx, count);
  if (st != ORACLE_OK) return st;
  int *clipped = (int *)malloc((size_t)B * Hkv * sizeof(int));
  if (!clipped) return ORACLE_NOMEM;
  for (int r = 0; r < B * Hkv; ++r) clipped[r] = count[r] < cap ? count[r] : cap;
  st = oracle_attn(L, B, Hq, Hkv, d, N, q_layers, K, V, idx, cap, clipped, out,
                   lse);
  free(clipped);
  return st;
}

/* Decode step with the routing set recomputed every R layers.  CLSA article,
 * section 計算コストの削減効果: per-layer routing (DSA) scores the context once
 * per layer, CLSA once per step; section 推論速度の改善結果: IndexCache shares
 * an index set across only some layers.  Reading: the L layers form groups
 * of R consecutive layers (the last group may be shorter); group g routes
 * with its own query q_routes[g] and its layers attend over that group's set.
 * R >= L is the shared-routing step above, R = 1 per-layer routing.
 * Layouts: q_routes [ngroups,B,Hq,d], tau [ngroups,B,Hkv] (threshold mode),
 * S [ngroups,B,Hkv,N], idx [ngroups,B,Hkv,stride], count [ngroups,B,Hkv],
 * out [L,B,Hq,d], lse [L,B,Hq]; ngroups = ceil(L/R). */
int oracle_decode_step_grouped(int L, int R, int B, int Hq, int Hkv, int d, int N,
                               const float *q_routes, const float *q_layers,
                               const float *K, const float *V, int k, const float *tau,
                               int cap, float *S, int *idx, int *count, double *out,
                               double *lse) {
  if (L < 1 || R < 1) return ORACLE_BAD_ARG;
  const int stride = k > 0 ? k : cap;
  const int ngroups = (L + R - 1) / R;
  for (int g = 0; g < ngroups; ++g) {
    const int l0 = g * R, lg = (L - l0) < R ? (L - l0) : R;
    const int st = oracle_decode_step(
        lg, B, Hq, Hkv, d, N, q_routes + (size_t)g * B * Hq * d,
        q_layers + (size_t)l0 * B * Hq * d, K, V, k,
        tau ? tau + (size_t)g * B * Hkv : NULL, cap, S + (size_t)g * B * Hkv * N,
        idx + (size_t)g * B * Hkv * stride, count + (size_t)g * B * Hkv,
        out + (size_t)l0 * B * Hq * d, lse + (size_t)l0 * B * Hq);
    if (st != ORACLE_OK) return st;
  }
  return ORACLE_OK;
}

#ifdef _OPENMP
#include <omp.h>
#endif
/* Threads the parallel loops above use (1 without OpenMP). */
int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
