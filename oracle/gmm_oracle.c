/*
 * gmm_oracle.c -- plain double-precision CPU reference for one EM step of a
 * diagonal-covariance Gaussian mixture.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle that the CUDA path is
 * checked against.  Only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark may load it.  It shares no code, header, table or helper
 * with the CUDA library, and the CUDA library never calls it.
 *
 * What it follows
 * ---------------
 * "Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering"
 * (review page, section 3 "Method & Key Results"): EM for a GMM in which an
 * E-step gives each point's responsibilities and the M-step is built from
 * sufficient statistics accumulated over all data tiles.  The pages name the
 * method but never print its formulas, so this file writes out the textbook
 * diagonal-covariance EM in direct form:
 *
 *   l_nk  = log pi_k - 1/2 sum_d [ log(2 pi var_kd) + (x_nd - mu_kd)^2 / var_kd ]
 *           (pi_k = 0  =>  l_nk = -inf)
 *   LSE_n = max_k l_nk + log sum_k exp(l_nk - max_k l_nk)
 *   r_nk  = exp(l_nk - LSE_n)
 *   LL    = sum_n LSE_n                      (log-likelihood of the INPUT params)
 *   N_k   = sum_n r_nk
 *   A_kd  = sum_n r_nk (x_nd - mu_kd)        (moments about the OLD mean: no
 *   B_kd  = sum_n r_nk (x_nd - mu_kd)^2       cancellation in the variance)
 *   pi'_k = N_k / N
 *   if N_k > 1e-12 N:  delta = A/N_k, mu' = mu + delta,
 *                      var' = max(B/N_k - delta^2, floor)
 *   else:              mu' = mu, var' = var  (empty component keeps its shape)
 *
 * Two loop-invariant hoists, both exact rearrangements of the formula above:
 * sum_d log(2 pi var_kd) is formed once per component, and 1/var_kd once per
 * element.  Nothing else is blocked, fused or reordered.
 *
 * Determinism: rows are cut into ORACLE_NBLOCKS fixed contiguous blocks; each
 * block accumulates privately; blocks are summed in block order.  Results do
 * not depend on the number of OpenMP threads.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_NBLOCKS 32

static const double ORACLE_LOG_2PI = 1.83787706640934548356065947281123527;

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Per-component quantities that do not depend on the point. */
typedef struct {
  int D, K;
  double* logw;    /* K: log pi_k, -inf when pi_k == 0 */
  double* logdet;  /* K: sum_d log(2 pi var_kd) */
  double* ivar;    /* K*D: 1 / var_kd */
} comp_consts;

static int consts_make(comp_consts* c, int D, int K, const double* w, const double* var) {
  c->D = D;
  c->K = K;
  c->logw = (double*)malloc(sizeof(double) * (size_t)K);
  c->logdet = (double*)malloc(sizeof(double) * (size_t)K);
  c->ivar = (double*)malloc(sizeof(double) * (size_t)K * (size_t)D);
  if (!c->logw || !c->logdet || !c->ivar) return -1;
  for (int k = 0; k < K; k++) {
    c->logw[k] = (w[k] > 0.0) ? log(w[k]) : -INFINITY;
    double s = 0.0;
    for (int d = 0; d < D; d++) {
      double v = var[(size_t)k * D + d];
      s += log(2.0 * M_PI * v);
      c->ivar[(size_t)k * D + d] = 1.0 / v;
    }
    c->logdet[k] = s;
  }
  return 0;
}

static void consts_free(comp_consts* c) {
  free(c->logw);
  free(c->logdet);
  free(c->ivar);
}

/* l_nk for one point x (length D) and every component; returns LSE_n. */
static double row_logjoint(const comp_consts* c, const double* x, const double* mu, double* l) {
  const int D = c->D, K = c->K;
  double m = -INFINITY;
  for (int k = 0; k < K; k++) {
    if (c->logw[k] == -INFINITY) {
      l[k] = -INFINITY;
      continue;
    }
    const double* mk = mu + (size_t)k * D;
    const double* ik = c->ivar + (size_t)k * D;
    double q = 0.0;
    for (int d = 0; d < D; d++) {
      double e = x[d] - mk[d];
      q += e * e * ik[d];
    }
    l[k] = c->logw[k] - 0.5 * (c->logdet[k] + q);
    if (l[k] > m) m = l[k];
  }
  double s = 0.0;
  for (int k = 0; k < K; k++) s += exp(l[k] - m);
  return m + log(s);
}

static void block_range(int64_t N, int b, int64_t* lo, int64_t* hi) {
  *lo = (N * b) / ORACLE_NBLOCKS;
  *hi = (N * (b + 1)) / ORACLE_NBLOCKS;
}

/*
 * E-step plus sufficient statistics about the old means.
 * Outputs: Nk[K], A[K*D], B[K*D], *loglik.  Returns 0, or -1 on allocation failure.
 */
int oracle_estep_stats(int64_t N, int D, int K, const double* X, const double* w,
                       const double* mu, const double* var, double* Nk, double* A,
                       double* B, double* loglik) {
  comp_consts c;
  if (consts_make(&c, D, K, w, var) != 0) {
    consts_free(&c);
    return -1;
  }
  const size_t stride = (size_t)K * (2 * (size_t)D + 1) + 1;
  double* part = (double*)calloc((size_t)ORACLE_NBLOCKS * stride, sizeof(double));
  if (!part) {
    consts_free(&c);
    return -1;
  }
  int fail = 0;
#pragma omp parallel
  {
    double* l = (double*)malloc(sizeof(double) * (size_t)K);
    if (!l) {
#pragma omp atomic write
      fail = 1;
    }
#pragma omp for schedule(dynamic, 1)
    for (int b = 0; b < ORACLE_NBLOCKS; b++) {
      if (!l) continue;
      double* pN = part + (size_t)b * stride;
      double* pA = pN + K;
      double* pB = pA + (size_t)K * D;
      double* pLL = pB + (size_t)K * D;
      int64_t lo, hi;
      block_range(N, b, &lo, &hi);
      for (int64_t n = lo; n < hi; n++) {
        const double* x = X + (size_t)n * D;
        double lse = row_logjoint(&c, x, mu, l);
        *pLL += lse;
        for (int k = 0; k < K; k++) {
          double r = exp(l[k] - lse);
          if (r == 0.0) continue; /* adding an exact zero changes nothing */
          pN[k] += r;
          const double* mk = mu + (size_t)k * D;
          double* ak = pA + (size_t)k * D;
          double* bk = pB + (size_t)k * D;
          for (int d = 0; d < D; d++) {
            double e = x[d] - mk[d];
            ak[d] += r * e;
            bk[d] += r * e * e;
          }
        }
      }
    }
    free(l);
  }
  if (!fail) {
    memset(Nk, 0, sizeof(double) * (size_t)K);
    memset(A, 0, sizeof(double) * (size_t)K * D);
    memset(B, 0, sizeof(double) * (size_t)K * D);
    double ll = 0.0;
    for (int b = 0; b < ORACLE_NBLOCKS; b++) {
      const double* pN = part + (size_t)b * stride;
      const double* pA = pN + K;
      const double* pB = pA + (size_t)K * D;
      for (int k = 0; k < K; k++) Nk[k] += pN[k];
      for (size_t i = 0; i < (size_t)K * D; i++) A[i] += pA[i];
      for (size_t i = 0; i < (size_t)K * D; i++) B[i] += pB[i];
      ll += pB[(size_t)K * D];
    }
    *loglik = ll;
  }
  free(part);
  consts_free(&c);
  return fail ? -1 : 0;
}

/* M-step from statistics about the old means (see the file header). */
void oracle_mstep(int64_t N, int D, int K, const double* mu, const double* var,
                  const double* Nk, const double* A, const double* B, double var_floor,
                  double* w_out, double* mu_out, double* var_out) {
  const double nmin = 1e-12 * (double)N;
  for (int k = 0; k < K; k++) {
    const double nk = Nk[k];
    w_out[k] = nk / (double)N;
    for (int d = 0; d < D; d++) {
      const size_t i = (size_t)k * D + d;
      if (nk > nmin) {
        const double delta = A[i] / nk;
        mu_out[i] = mu[i] + delta;
        const double v = B[i] / nk - delta * delta;
        var_out[i] = v > var_floor ? v : var_floor;
      } else {
        mu_out[i] = mu[i];
        var_out[i] = var[i];
      }
    }
  }
}

/* One EM step: theta -> theta', and LL(theta) (the input parameters). */
int oracle_em_step(int64_t N, int D, int K, const double* X, const double* w,
                   const double* mu, const double* var, double var_floor, double* w_out,
                   double* mu_out, double* var_out, double* loglik, double* Nk_out) {
  double* Nk = (double*)malloc(sizeof(double) * (size_t)K);
  double* A = (double*)malloc(sizeof(double) * (size_t)K * D);
  double* B = (double*)malloc(sizeof(double) * (size_t)K * D);
  int rc = -1;
  if (Nk && A && B) {
    rc = oracle_estep_stats(N, D, K, X, w, mu, var, Nk, A, B, loglik);
    if (rc == 0) {
      oracle_mstep(N, D, K, mu, var, Nk, A, B, var_floor, w_out, mu_out, var_out);
      if (Nk_out) memcpy(Nk_out, Nk, sizeof(double) * (size_t)K);
    }
  }
  free(Nk);
  free(A);
  free(B);
  return rc;
}

/* LL(theta) = sum_n LSE_n, with the same fixed block order as the E-step. */
int oracle_loglik(int64_t N, int D, int K, const double* X, const double* w,
                  const double* mu, const double* var, double* loglik) {
  comp_consts c;
  if (consts_make(&c, D, K, w, var) != 0) {
    consts_free(&c);
    return -1;
  }
  double part[ORACLE_NBLOCKS];
  memset(part, 0, sizeof(part));
  int fail = 0;
#pragma omp parallel
  {
    double* l = (double*)malloc(sizeof(double) * (size_t)K);
    if (!l) {
#pragma omp atomic write
      fail = 1;
    }
#pragma omp for schedule(dynamic, 1)
    for (int b = 0; b < ORACLE_NBLOCKS; b++) {
      if (!l) continue;
      int64_t lo, hi;
      block_range(N, b, &lo, &hi);
      double s = 0.0;
      for (int64_t n = lo; n < hi; n++) s += row_logjoint(&c, X + (size_t)n * D, mu, l);
      part[b] = s;
    }
    free(l);
  }
  double ll = 0.0;
  for (int b = 0; b < ORACLE_NBLOCKS; b++) ll += part[b];
  *loglik = ll;
  consts_free(&c);
  return fail ? -1 : 0;
}

/* Full responsibility matrix R[N*K] and LSE[N] (small N only: this is O(NK)). */
int oracle_responsibilities(int64_t N, int D, int K, const double* X, const double* w,
                            const double* mu, const double* var, double* R, double* lse) {
  comp_consts c;
  if (consts_make(&c, D, K, w, var) != 0) {
    consts_free(&c);
    return -1;
  }
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; n++) {
    double* l = R + (size_t)n * K;
    double s = row_logjoint(&c, X + (size_t)n * D, mu, l);
    if (lse) lse[n] = s;
    for (int k = 0; k < K; k++) l[k] = exp(l[k] - s);
  }
  consts_free(&c);
  return 0;
}

/*
 * Multi-assignment of each point to its m most responsible components
 * (Flash-GMM abstract: responsibilities assign border vectors to several
 * clusters).  Order: responsibility descending, equal values -> lower index.
 * Writes idx[N*m] and resp[N*m] (the responsibilities r_nk of those picks).
 */
int oracle_assign_topm(int64_t N, int D, int K, const double* X, const double* w,
                       const double* mu, const double* var, int m, int32_t* idx,
                       double* resp) {
  if (m < 1 || m > K) return -1;
  comp_consts c;
  if (consts_make(&c, D, K, w, var) != 0) {
    consts_free(&c);
    return -1;
  }
  int fail = 0;
#pragma omp parallel
  {
    double* l = (double*)malloc(sizeof(double) * (size_t)K);
    unsigned char* taken = (unsigned char*)malloc((size_t)K);
    if (!l || !taken) {
#pragma omp atomic write
      fail = 1;
    }
#pragma omp for schedule(static)
    for (int64_t n = 0; n < N; n++) {
      if (!l || !taken) continue;
      double s = row_logjoint(&c, X + (size_t)n * D, mu, l);
      for (int k = 0; k < K; k++) l[k] = exp(l[k] - s);
      memset(taken, 0, (size_t)K);
      for (int j = 0; j < m; j++) {
        int best = -1;
        for (int k = 0; k < K; k++) {
          if (taken[k]) continue;
          if (best < 0 || l[k] > l[best]) best = k; /* strict: ties keep the lower index */
        }
        taken[best] = 1;
        idx[(size_t)n * m + j] = best;
        resp[(size_t)n * m + j] = l[best];
      }
    }
    free(l);
    free(taken);
  }
  consts_free(&c);
  return fail ? -1 : 0;
}

/*
 * Initial parameters: means are the given K data rows, weights 1/K, and the
 * variances either 1 (var_mode 0) or the per-dimension biased sample variance
 * of X, floored (var_mode 1).  The row indices are an input: the caller draws
 * them.
 */
int oracle_init(int64_t N, int D, int K, const double* X, const int64_t* rows, int var_mode,
                double var_floor, double* w, double* mu, double* var) {
  for (int k = 0; k < K; k++) {
    if (rows[k] < 0 || rows[k] >= N) return -1;
    w[k] = 1.0 / (double)K;
    memcpy(mu + (size_t)k * D, X + (size_t)rows[k] * D, sizeof(double) * (size_t)D);
  }
  if (var_mode == 0) {
    for (size_t i = 0; i < (size_t)K * D; i++) var[i] = 1.0;
    return 0;
  }
  double* mean = (double*)calloc((size_t)D, sizeof(double));
  double* ss = (double*)calloc((size_t)D, sizeof(double));
  if (!mean || !ss) {
    free(mean);
    free(ss);
    return -1;
  }
  for (int64_t n = 0; n < N; n++)
    for (int d = 0; d < D; d++) mean[d] += X[(size_t)n * D + d];
  for (int d = 0; d < D; d++) mean[d] /= (double)N;
  for (int64_t n = 0; n < N; n++)
    for (int d = 0; d < D; d++) {
      double e = X[(size_t)n * D + d] - mean[d];
      ss[d] += e * e;
    }
  for (int k = 0; k < K; k++)
    for (int d = 0; d < D; d++) {
      double v = ss[d] / (double)N;
      var[(size_t)k * D + d] = v > var_floor ? v : var_floor;
    }
  free(mean);
  free(ss);
  return 0;
}

/* iters EM steps from the given parameters, in place; ll_hist[t] = LL(theta_t). */
int oracle_fit(int64_t N, int D, int K, const double* X, int iters, double var_floor,
               double* w, double* mu, double* var, double* ll_hist) {
  double* w2 = (double*)malloc(sizeof(double) * (size_t)K);
  double* mu2 = (double*)malloc(sizeof(double) * (size_t)K * D);
  double* var2 = (double*)malloc(sizeof(double) * (size_t)K * D);
  int rc = (w2 && mu2 && var2) ? 0 : -1;
  for (int t = 0; t < iters && rc == 0; t++) {
    rc = oracle_em_step(N, D, K, X, w, mu, var, var_floor, w2, mu2, var2, &ll_hist[t], NULL);
    if (rc == 0) {
      memcpy(w, w2, sizeof(double) * (size_t)K);
      memcpy(mu, mu2, sizeof(double) * (size_t)K * D);
      memcpy(var, var2, sizeof(double) * (size_t)K * D);
    }
  }
  free(w2);
  free(mu2);
  free(var2);
  return rc;
}

double oracle_log_2pi(void) { return ORACLE_LOG_2PI; }
