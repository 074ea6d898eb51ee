/*
 * streamkl_oracle.c -- plain fp64 CPU oracle for the row-wise attention KL
 * divergence KL(P1 || P2) and its gradients.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only tests/, the smoke check and the benchmark's CPU
 * baseline do.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes (StreamKL summary page, "Metodologia" section 1 and 2):
 *
 *   x1[i,j] = s1 * <Q1[i], K1[j]>,   x2[i,j] = s2 * <Q2[i], K2[j]>
 *   P_t[i,:] = softmax over the visible keys J_i of x_t[i,:]
 *   LSE_t[i] = log sum_{j in J_i} exp(x_t[i,j])            ("LSE_t = m_t + log l_t")
 *   L[i]     = sum_{j in J_i} P1[i,j] * ((x1 - LSE1) - (x2 - LSE2))  = KL(P1_i || P2_i)
 *
 * The page reaches this exact value with an online five-scalar recurrence;
 * the oracle does not: it writes the definition out, materialising one row of
 * logits at a time (two passes: max, then sum of exponentials).  The log ratio
 * is formed from logit differences and the LSEs, never as log(P1/P2), which is
 * the numerically stable form the page asks for in "Stabilita Numerica".
 *
 * Backward (section 2, "Strategia di Ricalcolo", both gradient
 * configurations): with upstream weight g_i on L_i, differentiating the
 * definition gives
 *
 *   dS1[i,j] = g_i * P1[i,j] * ((x1 - LSE1) - (x2 - LSE2) - L_i)
 *   dS2[i,j] = g_i * (P2[i,j] - P1[i,j])
 *   dQ_t[i] = s_t * sum_j dS_t[i,j] K_t[j],   dK_t[j] = s_t * sum_i dS_t[i,j] Q_t[i]
 *
 * Masked pairs contribute nothing.  Causal visibility is bottom-right aligned:
 * key j is visible from query row i when j <= i + NK - NQ (the usual j <= i when
 * NQ == NK).
 *
 * Inputs are either bf16 bit patterns (decoded exactly to double) or doubles,
 * laid out contiguous [BH][N][d].  Rows are independent, so work is split
 * over POSIX threads by row; per-thread dK partial sums are added in thread
 * order at the end, so results do not depend on scheduling.
 *
 * Planted-mistake builds: compiling with -DORACLE_MUTANT=k (k >= 1) plants one
 * deliberate error so that the tests can show their pins catch it.  The
 * default build (no macro) is the oracle.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

typedef struct {
  int64_t BH, NQ, NK;
  int d1, d2, causal, in_bf16;
  double s1, s2;
  const void *Q1, *K1, *Q2, *K2;
} problem_t;

/* bf16 is the top half of an IEEE binary32; the decode is exact. */
static inline double ld(const void *base, int in_bf16, int64_t idx) {
  if (in_bf16) {
    uint32_t u = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
  }
  return ((const double *)base)[idx];
}

/* Number of keys visible from query row i (keys 0 .. count-1). */
static int64_t visible_keys(const problem_t *p, int64_t i) {
  if (!p->causal) return p->NK;
  int64_t v = i + p->NK - p->NQ + 1;
#if ORACLE_MUTANT == 4
  v -= 1; /* planted: causal frontier off by one */
#endif
  if (v < 0) v = 0;
  if (v > p->NK) v = p->NK;
  return v;
}

/* Logits of one row: x[j] = s * <Q[bh,i,:], K[bh,j,:]> for j < nvis. */
static void row_logits(const void *Q, const void *K, int in_bf16, int64_t NQ, int64_t NK, int d,
                       double s, int64_t bh, int64_t i, int64_t nvis, double *q, double *x) {
  int64_t qoff = (bh * NQ + i) * d;
  for (int k = 0; k < d; ++k) q[k] = ld(Q, in_bf16, qoff + k);
  for (int64_t j = 0; j < nvis; ++j) {
    int64_t koff = (bh * NK + j) * d;
    double acc = 0.0;
    for (int k = 0; k < d; ++k) {
#if ORACLE_MUTANT == 3
      /* planted: transposed key operand (reads K[k][j] instead of K[j][k]) */
      int64_t kk = (bh * NK + (k % NK)) * d + (int)(j % d);
      acc += q[k] * ld(K, in_bf16, kk);
#else
      acc += q[k] * ld(K, in_bf16, koff + k);
#endif
    }
    x[j] = s * acc;
  }
}

/* log sum_j exp(x[j]) by the two-pass max shift. */
static double logsumexp(const double *x, int64_t n) {
  if (n == 0) return -INFINITY;
  double m = x[0];
  for (int64_t j = 1; j < n; ++j)
    if (x[j] > m) m = x[j];
  double sum = 0.0;
  for (int64_t j = 0; j < n; ++j) sum += exp(x[j] - m);
  return m + log(sum);
}

/* Row statistics from materialised logit rows x1, x2 of length n. */
static void row_stats(const double *x1, const double *x2, int64_t n, double *L, double *lse1,
                      double *lse2) {
  double a = logsumexp(x1, n), b = logsumexp(x2, n);
  double kl = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    double lp1 = x1[j] - a, lp2 = x2[j] - b;
#if ORACLE_MUTANT == 1
    lp2 = x2[j]; /* planted: LSE2 term dropped from the log ratio */
#endif
    kl += exp(lp1) * (lp1 - lp2);
  }
  *L = kl;
  *lse1 = a;
  *lse2 = b;
}

/* ---- threading ---------------------------------------------------------- */

typedef struct {
  const problem_t *p;
  int64_t lo, hi; /* this thread's slice of the work list */
  const int64_t *rows;
  const double *g;
  double *L, *LSE1, *LSE2, *dQ1, *dQ2;
  double *dK1, *dK2; /* per-thread partials for the head variant */
  int64_t head;      /* head variant: bh of the head */
  int status;
} job_t;

static int run_threads(void *(*fn)(void *), job_t *jobs, int nthreads) {
  if (nthreads <= 1) {
    fn(&jobs[0]);
    return jobs[0].status;
  }
  pthread_t *t = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
  char *made = (char *)calloc((size_t)nthreads, 1);
  if (!t || !made) {
    free(t); free(made);
    return -1;
  }
  for (int k = 0; k < nthreads; ++k) {
    if (pthread_create(&t[k], NULL, fn, &jobs[k]) == 0)
      made[k] = 1;
    else
      fn(&jobs[k]); /* could not start a thread: run the slice here */
  }
  for (int k = 0; k < nthreads; ++k)
    if (made[k]) pthread_join(t[k], NULL);
  free(t); free(made);
  int st = 0;
  for (int k = 0; k < nthreads; ++k)
    if (jobs[k].status) st = jobs[k].status;
  return st;
}

static int clamp_threads(int nthreads, int64_t work) {
  if (nthreads < 1) nthreads = 1;
  if (work < nthreads) nthreads = (int)(work > 0 ? work : 1);
  return nthreads;
}

/* ---- forward over a list of rows ---------------------------------------- */

static void *fwd_rows_worker(void *arg) {
  job_t *jb = (job_t *)arg;
  const problem_t *p = jb->p;
  int dmax = p->d1 > p->d2 ? p->d1 : p->d2;
  double *q = (double *)malloc(sizeof(double) * (size_t)dmax);
  double *x1 = (double *)malloc(sizeof(double) * (size_t)(p->NK > 0 ? p->NK : 1));
  double *x2 = (double *)malloc(sizeof(double) * (size_t)(p->NK > 0 ? p->NK : 1));
  if (!q || !x1 || !x2) {
    jb->status = -1;
    free(q); free(x1); free(x2);
    return NULL;
  }
  for (int64_t r = jb->lo; r < jb->hi; ++r) {
    int64_t bh = jb->rows[2 * r], i = jb->rows[2 * r + 1];
    int64_t n = visible_keys(p, i);
    row_logits(p->Q1, p->K1, p->in_bf16, p->NQ, p->NK, p->d1, p->s1, bh, i, n, q, x1);
    row_logits(p->Q2, p->K2, p->in_bf16, p->NQ, p->NK, p->d2, p->s2, bh, i, n, q, x2);
    row_stats(x1, x2, n, &jb->L[r], &jb->LSE1[r], &jb->LSE2[r]);
  }
  free(q); free(x1); free(x2);
  return NULL;
}

static int check_problem(const problem_t *p) {
  if (p->BH < 1 || p->NQ < 1 || p->NK < 1 || p->d1 < 1 || p->d2 < 1) return 1;
  if (!p->Q1 || !p->K1 || !p->Q2 || !p->K2) return 1;
  return 0;
}

/*
 * Forward on nrows listed rows.  rows holds (bh, i) pairs.  L, LSE1 and LSE2
 * receive one value per listed row.  Returns 0 on success, 1 on a bad
 * argument, -1 if memory ran out.
 */
int oracle_fwd_rows(int64_t BH, int64_t NQ, int64_t NK, int d1, int d2, int causal, double s1,
                    double s2, int in_bf16, const void *Q1, const void *K1, const void *Q2,
                    const void *K2, int64_t nrows, const int64_t *rows, double *L, double *LSE1,
                    double *LSE2, int nthreads) {
  problem_t p = {BH, NQ, NK, d1, d2, causal, in_bf16, s1, s2, Q1, K1, Q2, K2};
  if (check_problem(&p) || nrows < 0 || (nrows > 0 && (!rows || !L || !LSE1 || !LSE2))) return 1;
  for (int64_t r = 0; r < nrows; ++r)
    if (rows[2 * r] < 0 || rows[2 * r] >= BH || rows[2 * r + 1] < 0 || rows[2 * r + 1] >= NQ)
      return 1;
  if (nrows == 0) return 0;
  nthreads = clamp_threads(nthreads, nrows);
  job_t *jobs = (job_t *)calloc((size_t)nthreads, sizeof(job_t));
  if (!jobs) return -1;
  for (int k = 0; k < nthreads; ++k) {
    jobs[k].p = &p;
    jobs[k].lo = nrows * k / nthreads;
    jobs[k].hi = nrows * (k + 1) / nthreads;
    jobs[k].rows = rows;
    jobs[k].L = L; jobs[k].LSE1 = LSE1; jobs[k].LSE2 = LSE2;
  }
  int st = run_threads(fwd_rows_worker, jobs, nthreads);
  free(jobs);
  return st;
}

/* ---- backward ----------------------------------------------------------- */

/*
 * Per row: recompute the logits, the statistics, then dS1/dS2 and accumulate
 * dQ (always) and, when dK1/dK2 are given, the dK partials of this thread.
 */
static int bwd_one_row(const problem_t *p, int64_t bh, int64_t i, double g, double *q1, double *q2,
                       double *x1, double *x2, double *Lo, double *l1o, double *l2o, double *dq1,
                       double *dq2, double *dK1, double *dK2) {
  int64_t n = visible_keys(p, i);
  row_logits(p->Q1, p->K1, p->in_bf16, p->NQ, p->NK, p->d1, p->s1, bh, i, n, q1, x1);
  row_logits(p->Q2, p->K2, p->in_bf16, p->NQ, p->NK, p->d2, p->s2, bh, i, n, q2, x2);
  double L, a, b;
  row_stats(x1, x2, n, &L, &a, &b);
  *Lo = L; *l1o = a; *l2o = b;
  for (int k = 0; k < p->d1; ++k) dq1[k] = 0.0;
  for (int k = 0; k < p->d2; ++k) dq2[k] = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    double lp1 = x1[j] - a, lp2 = x2[j] - b;
    double P1 = exp(lp1), P2 = exp(lp2);
    double ds1 = g * P1 * (lp1 - lp2 - L);
#if ORACLE_MUTANT == 5
    ds1 = g * P1 * (x1[j] - x2[j] - L); /* planted: raw-logit reading of dL/dx1 */
#endif
    double ds2 = g * (P2 - P1);
#if ORACLE_MUTANT == 2
    ds2 = -ds2; /* planted: wrong sign of dL/dx2 */
#endif
    int64_t k1off = (bh * p->NK + j) * p->d1, k2off = (bh * p->NK + j) * p->d2;
    for (int k = 0; k < p->d1; ++k) dq1[k] += p->s1 * ds1 * ld(p->K1, p->in_bf16, k1off + k);
    for (int k = 0; k < p->d2; ++k) dq2[k] += p->s2 * ds2 * ld(p->K2, p->in_bf16, k2off + k);
    if (dK1) {
      for (int k = 0; k < p->d1; ++k) dK1[j * p->d1 + k] += p->s1 * ds1 * q1[k];
      for (int k = 0; k < p->d2; ++k) dK2[j * p->d2 + k] += p->s2 * ds2 * q2[k];
    }
  }
  return 0;
}

static void *bwd_rows_worker(void *arg) {
  job_t *jb = (job_t *)arg;
  const problem_t *p = jb->p;
  size_t nk = (size_t)(p->NK > 0 ? p->NK : 1);
  double *q1 = (double *)malloc(sizeof(double) * (size_t)p->d1);
  double *q2 = (double *)malloc(sizeof(double) * (size_t)p->d2);
  double *x1 = (double *)malloc(sizeof(double) * nk);
  double *x2 = (double *)malloc(sizeof(double) * nk);
  if (!q1 || !q2 || !x1 || !x2) {
    jb->status = -1;
    free(q1); free(q2); free(x1); free(x2);
    return NULL;
  }
  for (int64_t r = jb->lo; r < jb->hi; ++r) {
    int64_t bh, i;
    double g;
    double *dq1, *dq2;
    if (jb->rows) { /* row-list variant */
      bh = jb->rows[2 * r]; i = jb->rows[2 * r + 1]; g = jb->g[r];
      dq1 = jb->dQ1 + r * p->d1; dq2 = jb->dQ2 + r * p->d2;
    } else { /* whole-head variant: r is the row index within head jb->head */
      bh = jb->head; i = r; g = jb->g[r];
      dq1 = jb->dQ1 + r * p->d1; dq2 = jb->dQ2 + r * p->d2;
    }
    bwd_one_row(p, bh, i, g, q1, q2, x1, x2, &jb->L[r], &jb->LSE1[r], &jb->LSE2[r], dq1, dq2,
                jb->dK1, jb->dK2);
  }
  free(q1); free(q2); free(x1); free(x2);
  return NULL;
}

/*
 * Backward on listed rows: for each (bh, i) in rows with upstream weight g[r],
 * writes L, LSE1, LSE2 and the query gradients dQ1 [nrows][d1], dQ2
 * [nrows][d2].  Key gradients need every row of a head: see
 * oracle_bwd_heads.
 */
int oracle_bwd_rows(int64_t BH, int64_t NQ, int64_t NK, int d1, int d2, int causal, double s1,
                    double s2, int in_bf16, const void *Q1, const void *K1, const void *Q2,
                    const void *K2, int64_t nrows, const int64_t *rows, const double *g, double *L,
                    double *LSE1, double *LSE2, double *dQ1, double *dQ2, int nthreads) {
  problem_t p = {BH, NQ, NK, d1, d2, causal, in_bf16, s1, s2, Q1, K1, Q2, K2};
  if (check_problem(&p) || nrows < 0) return 1;
  if (nrows > 0 && (!rows || !g || !L || !LSE1 || !LSE2 || !dQ1 || !dQ2)) return 1;
  for (int64_t r = 0; r < nrows; ++r)
    if (rows[2 * r] < 0 || rows[2 * r] >= BH || rows[2 * r + 1] < 0 || rows[2 * r + 1] >= NQ)
      return 1;
  if (nrows == 0) return 0;
  nthreads = clamp_threads(nthreads, nrows);
  job_t *jobs = (job_t *)calloc((size_t)nthreads, sizeof(job_t));
  if (!jobs) return -1;
  for (int k = 0; k < nthreads; ++k) {
    jobs[k].p = &p;
    jobs[k].lo = nrows * k / nthreads;
    jobs[k].hi = nrows * (k + 1) / nthreads;
    jobs[k].rows = rows; jobs[k].g = g;
    jobs[k].L = L; jobs[k].LSE1 = LSE1; jobs[k].LSE2 = LSE2;
    jobs[k].dQ1 = dQ1; jobs[k].dQ2 = dQ2;
  }
  int st = run_threads(bwd_rows_worker, jobs, nthreads);
  free(jobs);
  return st;
}

/*
 * Backward on whole heads.  heads lists nheads values of bh.  g is
 * [nheads][NQ].  Outputs: L, LSE1, LSE2 [nheads][NQ]; dQ1 [nheads][NQ][d1],
 * dK1 [nheads][NK][d1], dQ2 [nheads][NQ][d2], dK2 [nheads][NK][d2].
 */
int oracle_bwd_heads(int64_t BH, int64_t NQ, int64_t NK, int d1, int d2, int causal, double s1,
                     double s2, int in_bf16, const void *Q1, const void *K1, const void *Q2,
                     const void *K2, int64_t nheads, const int64_t *heads, const double *g,
                     double *L, double *LSE1, double *LSE2, double *dQ1, double *dK1, double *dQ2,
                     double *dK2, int nthreads) {
  problem_t p = {BH, NQ, NK, d1, d2, causal, in_bf16, s1, s2, Q1, K1, Q2, K2};
  if (check_problem(&p) || nheads < 0) return 1;
  if (nheads > 0 && (!heads || !g || !L || !LSE1 || !LSE2 || !dQ1 || !dK1 || !dQ2 || !dK2))
    return 1;
  for (int64_t h = 0; h < nheads; ++h)
    if (heads[h] < 0 || heads[h] >= BH) return 1;
  int T = clamp_threads(nthreads, NQ);
  job_t *jobs = (job_t *)calloc((size_t)T, sizeof(job_t));
  if (!jobs) return -1;
  size_t kd1 = (size_t)NK * (size_t)d1, kd2 = (size_t)NK * (size_t)d2;
  double *part1 = (double *)calloc((size_t)T * kd1, sizeof(double));
  double *part2 = (double *)calloc((size_t)T * kd2, sizeof(double));
  if (!part1 || !part2) {
    free(jobs); free(part1); free(part2);
    return -1;
  }
  int st = 0;
  for (int64_t h = 0; h < nheads && st == 0; ++h) {
    memset(part1, 0, sizeof(double) * (size_t)T * kd1);
    memset(part2, 0, sizeof(double) * (size_t)T * kd2);
    for (int k = 0; k < T; ++k) {
      memset(&jobs[k], 0, sizeof(job_t));
      jobs[k].p = &p;
      jobs[k].lo = NQ * k / T;
      jobs[k].hi = NQ * (k + 1) / T;
      jobs[k].head = heads[h];
      jobs[k].g = g + h * NQ;
      jobs[k].L = L + h * NQ; jobs[k].LSE1 = LSE1 + h * NQ; jobs[k].LSE2 = LSE2 + h * NQ;
      jobs[k].dQ1 = dQ1 + h * NQ * d1; jobs[k].dQ2 = dQ2 + h * NQ * d2;
      jobs[k].dK1 = part1 + (size_t)k * kd1;
      jobs[k].dK2 = part2 + (size_t)k * kd2;
    }
    st = run_threads(bwd_rows_worker, jobs, T);
    double *o1 = dK1 + (size_t)h * kd1, *o2 = dK2 + (size_t)h * kd2;
    for (size_t e = 0; e < kd1; ++e) {
      double s = 0.0;
      for (int k = 0; k < T; ++k) s += part1[(size_t)k * kd1 + e];
      o1[e] = s;
    }
    for (size_t e = 0; e < kd2; ++e) {
      double s = 0.0;
      for (int k = 0; k < T; ++k) s += part2[(size_t)k * kd2 + e];
      o2[e] = s;
    }
  }
  free(jobs); free(part1); free(part2);
  return st;
}

/* Build identification, so tests can tell a planted-mistake build apart. */
int oracle_mutant_id(void) { return ORACLE_MUTANT; }
