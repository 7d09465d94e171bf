// mstep_init.cuh -- the M-step from canonical statistics, and the seeded
// initialisation's gather and data-moment kernels.
//
// Method: "Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering"
// (review page, section 3): the per-tile statistics, accumulated globally,
// feed the M-step; the M-step itself is the textbook diagonal one (the pages
// leave it implicit).
#pragma once

#include <math.h>

#include "common.cuh"

namespace scem {

// M-step from canonical statistics of `nshards` disjoint row shards
// (consecutive buffers of K(2D+1)+1 doubles, summed here in shard order) of N
// points in total: pi_k = N_k / N; if N_k > 1e-12 N: delta = A/N_k,
// mu += delta, var = max(B/N_k - delta^2, floor); else mu and var are kept.
__global__ void __launch_bounds__(256) mstep_kernel(int64_t N, int D, int K, float var_floor,
                                                    const double* __restrict__ stats, int nshards,
                                                    float* __restrict__ w, float* __restrict__ mu,
                                                    float* __restrict__ var,
                                                    double* __restrict__ loglik) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t KD = (size_t)K * D;
  const size_t S = (size_t)K + 2 * KD + 1;
  if (i == 0 && loglik) {
    double ll = 0.0;
    for (int s = 0; s < nshards; s++) ll += stats[(size_t)s * S + K + 2 * KD];
    *loglik = ll;
  }
  if (i >= KD) return;
  const int k = (int)(i / D);
  double nk = 0.0, a = 0.0, b = 0.0;
  for (int s = 0; s < nshards; s++) {
    const double* st = stats + (size_t)s * S;
    nk += st[k];
    a += st[K + i];
    b += st[K + KD + i];
  }
  if (i - (size_t)k * D == 0) w[k] = (float)(nk / (double)N);
  if (nk > 1e-12 * (double)N) {
    const double delta = a / nk;
    double v = b / nk - delta * delta;
    if (!(v > (double)var_floor)) v = (double)var_floor;
    mu[i] = (float)((double)mu[i] + delta);
    var[i] = (float)v;
  }
}

// ---------------------------------------------------------------------------
// Init: means from the chosen rows, weights 1/K, and per-dimension data
// moments (two fixed-order fp64 passes: mean, then mean squared deviation).
// ---------------------------------------------------------------------------
template <typename XT>
__global__ void init_gather_kernel(const XT* __restrict__ X, int D, int K,
                                   const int64_t* __restrict__ rows, int var_mode,
                                   float* __restrict__ w, float* __restrict__ mu,
                                   float* __restrict__ var) {
  const int k = blockIdx.x;
  const int64_t r = rows[k];
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    mu[(size_t)k * D + d] = load_x(X, (size_t)r * D + d);
    if (var_mode == GMM_INIT_VAR_ONE) var[(size_t)k * D + d] = 1.0f;
  }
  if (threadIdx.x == 0) w[k] = (float)(1.0 / (double)K);
}

// Partial column sums over the row block of CTA p: sum x (mean == NULL) or
// sum (x - mean)^2.  part is P x D.
template <typename XT>
__global__ void __launch_bounds__(256) col_partial_kernel(const XT* __restrict__ X, int64_t N,
                                                          int D, const double* __restrict__ mean,
                                                          double* __restrict__ part) {
  __shared__ double red[256];
  const int P = gridDim.x, p = blockIdx.x, tid = threadIdx.x;
  const int64_t lo = N * p / P, hi = N * (p + 1) / P;
  if (D <= 256) {
    const int rpi = 256 / D, roff = tid / D, d = tid - roff * D;
    double s = 0.0;
    if (roff < rpi)
      for (int64_t n = lo + roff; n < hi; n += rpi) {
        const double x = (double)load_x(X, (size_t)n * D + d);
        s += mean ? (x - mean[d]) * (x - mean[d]) : x;
      }
    red[tid] = s;
    __syncthreads();
    if (tid < D) {
      double t = 0.0;
      for (int q = 0; q < rpi; q++) t += red[q * D + tid];
      part[(size_t)p * D + tid] = t;
    }
  } else {
    for (int d = tid; d < D; d += 256) {
      double s = 0.0;
      for (int64_t n = lo; n < hi; n++) {
        const double x = (double)load_x(X, (size_t)n * D + d);
        s += mean ? (x - mean[d]) * (x - mean[d]) : x;
      }
      part[(size_t)p * D + d] = s;
    }
  }
}

// Fixed-order sum of the P partials.  pass 0: out[d] = mean.  pass 1: the
// floored variance, written to every component's row of var.
__global__ void col_finish_kernel(int64_t N, int D, int K, int P, const double* __restrict__ part,
                                  int pass, float var_floor, double* __restrict__ mean_out,
                                  float* __restrict__ var) {
  const int d = blockIdx.x * blockDim.x + threadIdx.x;
  if (d >= D) return;
  double s = 0.0;
  for (int p = 0; p < P; p++) s += part[(size_t)p * D + d];
  s /= (double)N;
  if (pass == 0) {
    mean_out[d] = s;
  } else {
    const float v = (s > (double)var_floor) ? (float)s : var_floor;
    for (int k = 0; k < K; k++) var[(size_t)k * D + d] = v;
  }
}

}  // namespace scem
