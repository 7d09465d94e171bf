// variants.cuh -- the M-steps and parameter set-up of three neighbours of the
// diagonal EM step, which share its fused E-step and statistics pass.
//
// "Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering" presents
// the soft mixture as a replacement for k-means in an IVF coarse quantizer
// (abstract; review page, section 3, k-means as the baseline).  The pages print
// none of these forms; they are the textbook ones:
//   spherical EM: covariance s2_k * I.  The E-step is the diagonal one with
//     var_kd = s2_k for every d (sph_expand_kernel); the M-step averages the
//     per-dimension variance about the new mean over the dimensions
//     (sph_mstep_kernel).
//   hard EM: the diagonal model with one-hot responsibilities (the fused
//     pass's hard mode); the diagonal M-step.
//   k-means: hard EM with equal weights and one variance v shared by every
//     component and dimension, so the most probable component is the nearest
//     centre in squared Euclidean distance (km_prep_kernel); the M-step moves
//     each centre to the mean of its points and keeps the rest
//     (km_mstep_kernel).
// Statistics are the canonical [N_k | A | B | LL] about the step's input means.
#pragma once

#include <math.h>

#include "common.cuh"

namespace scem {

// var[k][d] = s2[k]
__global__ void __launch_bounds__(256) sph_expand_kernel(int D, int K, const float* __restrict__ s2,
                                                         float* __restrict__ var) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < (size_t)K * D) var[i] = s2[i / D];
}

// One block per component: pi_k = N_k / N; if N_k > 1e-12 N, delta = A/N_k,
// mu' = mu + delta and s2' = max(mean_d(B/N_k - delta^2), floor) (the mean over
// d summed in a fixed tree order), else mu and s2 are kept.
__global__ void __launch_bounds__(128) sph_mstep_kernel(int64_t N, int D, int K, float var_floor,
                                                        const double* __restrict__ stats,
                                                        float* __restrict__ w,
                                                        float* __restrict__ mu,
                                                        float* __restrict__ s2,
                                                        double* __restrict__ loglik) {
  __shared__ double red[128];
  const int k = blockIdx.x;
  const size_t KD = (size_t)K * D;
  const double nk = stats[k];
  const bool live = nk > 1e-12 * (double)N;
  double v = 0.0;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    const size_t i = (size_t)k * D + d;
    if (live) {
      const double delta = stats[K + i] / nk;
      v += stats[K + KD + i] / nk - delta * delta;
      mu[i] = (float)((double)mu[i] + delta);
    }
  }
  red[threadIdx.x] = v;
  __syncthreads();
  for (int s = 64; s > 0; s >>= 1) {
    if ((int)threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    w[k] = (float)(nk / (double)N);
    if (live) {
      double m = red[0] / (double)D;
      if (!(m > (double)var_floor)) m = (double)var_floor;
      s2[k] = (float)m;
    }
    if (k == 0 && loglik) *loglik = stats[K + 2 * KD];
  }
}

// Equal weights 1/K and one variance for every component and dimension: the
// average over dimensions of the centres' spread, v = (1/D) sum_d (1/K)
// sum_k (c_kd - cbar_d)^2 (1 if that is not positive).  Any shared v > 0 gives
// the same nearest centres; this one keeps the E-step's numbers in range.
// One block; *v_out receives v.
__global__ void __launch_bounds__(256) km_prep_kernel(int D, int K, const float* __restrict__ C,
                                                      float* __restrict__ w,
                                                      float* __restrict__ var,
                                                      float* __restrict__ v_out) {
  __shared__ double red[256];
  double s = 0.0;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    double m = 0.0, q = 0.0;
    for (int k = 0; k < K; k++) m += (double)C[(size_t)k * D + d];
    m /= K;
    for (int k = 0; k < K; k++) {
      const double e = (double)C[(size_t)k * D + d] - m;
      q += e * e;
    }
    s += q / K;
  }
  red[threadIdx.x] = s;
  __syncthreads();
  for (int h = 128; h > 0; h >>= 1) {
    if ((int)threadIdx.x < h) red[threadIdx.x] += red[threadIdx.x + h];
    __syncthreads();
  }
  float v = (float)(red[0] / D);
  if (!(v > 0.f) || !isfinite(v)) v = 1.0f;
  for (int k = threadIdx.x; k < K; k += blockDim.x) w[k] = 1.0f / (float)K;
  for (size_t i = threadIdx.x; i < (size_t)K * D; i += blockDim.x) var[i] = v;
  if (threadIdx.x == 0) *v_out = v;
}

// Centres to the mean of their points (c' = c + A/N_k where N_k > 0, else
// kept), and the inertia of the input centres, sum_n min_k |x_n - c_k|^2,
// from the classification log-likelihood LL = sum_n max_k l_nk of the model
// l_nk = log(1/K) - (D/2) log(2 pi v) - |x_n - c_k|^2 / (2 v):
//   inertia = -2 v (LL - N (log(1/K) - (D/2) log(2 pi v))).
__global__ void __launch_bounds__(256) km_mstep_kernel(int64_t N, int D, int K,
                                                       const double* __restrict__ stats,
                                                       const float* __restrict__ v_in,
                                                       float* __restrict__ C,
                                                       double* __restrict__ inertia) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t KD = (size_t)K * D;
  if (i == 0 && inertia) {
    const double v = (double)*v_in;
    const double c0 = log(1.0 / (double)K) - 0.5 * D * log(2.0 * M_PI * v);
    *inertia = -2.0 * v * (stats[K + 2 * KD] - (double)N * c0);
  }
  if (i >= KD) return;
  const double nk = stats[i / D];
  if (nk > 0.5) C[i] = (float)((double)C[i] + stats[K + i] / nk);
}

}  // namespace scem
