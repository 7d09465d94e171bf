// small_fit.cuh -- gmm_fit in one launch for problems whose data fit in the
// shared memory of one thread-block cluster.
//
// Method: "Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering"
// (review page, section 3): every EM iteration is an E-step over the data,
// per-point normalisation into responsibilities, sufficient statistics summed
// over all points, then the M-step.  For a small problem (the 10^4-point,
// 16-dimension, 8-component mixture) the cost of an iteration is launch and
// synchronisation latency, not arithmetic, so all iterations run inside one
// launch of one cluster: the cluster's CTAs hold disjoint row blocks of X in
// shared memory for the whole fit, exchange their per-iteration statistics
// over distributed shared memory, and each applies the same M-step.
//
// Per iteration, in each CTA:
//   1. rows (one thread per row at a time; X and r are stored dimension- and
//      component-major, [d][n] and [k][n], so a warp's rows are consecutive
//      words): l_k = c_k - 1/2 sum_d (x_d - mu_kd)^2
//      / var_kd in fp32, direct form (c_k = log pi_k - 1/2 sum_d log(2 pi var_kd),
//      -inf for pi_k = 0), LSE = max + log sum exp, r_k = exp(l_k - LSE), kept
//      in shared memory; LL partial += LSE in fp64.
//   2. statistics about the iteration's input means, one (k, d) pair per
//      thread over the CTA's rows in row order, fp64: N_k = sum r, A_kd =
//      sum r (x - mu), B_kd = sum r (x - mu)^2, into this iteration's partial
//      buffer (two buffers alternate).
//   3. cluster barrier; every CTA sums the C partials in CTA order (DSMEM
//      loads), so all hold the same totals, and applies the M-step: pi = N_k/N;
//      if N_k > 1e-12 N, delta = A/N_k, mu' = mu + delta, var' = max(B/N_k -
//      delta^2, floor), else mu and var are kept.  CTA 0 records LL of the
//      iteration's input parameters.
// The alternating partial buffers need one cluster barrier per iteration: a
// CTA writes buffer t % 2 only after the barrier of iteration t - 1, which
// every CTA reaches after it has read buffer (t - 2) % 2 = t % 2.
#pragma once

#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "sm100_prims.cuh"
#include "tc_em.cuh"  // load1

namespace scem {

constexpr int kSfThreads = 256;
constexpr int kSfMaxCluster = 16;
constexpr uint32_t kSfMaxSmem = 200 * 1024;

// Shared-memory layout (byte offsets) of the small-fit kernel for C CTAs.
struct SfLayout {
  uint32_t x, r, w, mu, var, iv, cst, part, tot, red, total;
  int64_t rows;  // rows per CTA (the last CTA may hold fewer)
};

__host__ __device__ inline uint32_t sf_align(uint32_t v) { return (v + 15u) & ~15u; }

__host__ __device__ inline SfLayout sf_layout(int64_t N, int D, int K, int C) {
  SfLayout L;
  L.rows = (N + C - 1) / C;
  const uint32_t S = (uint32_t)K * (2u * D + 1u) + 1u;  // [N_k | A | B | LL]
  uint32_t off = 0;
  L.x = off;
  off = sf_align(off + (uint32_t)(L.rows * D * 4));
  L.r = off;
  off = sf_align(off + (uint32_t)(L.rows * K * 4));
  L.w = off;
  off = sf_align(off + (uint32_t)K * 4);
  L.mu = off;
  off = sf_align(off + (uint32_t)(K * D * 4));
  L.var = off;
  off = sf_align(off + (uint32_t)(K * D * 4));
  L.iv = off;
  off = sf_align(off + (uint32_t)(K * D * 4));
  L.cst = off;
  off = sf_align(off + (uint32_t)K * 4);
  L.part = off;
  off = sf_align(off + 2u * S * 8u);
  L.tot = off;
  off = sf_align(off + S * 8u);
  L.red = off;
  off = sf_align(off + kSfThreads * 8u);
  L.total = off;
  return L;
}

// Cluster size for a small fit: enough CTAs that a CTA holds at most ~640 rows,
// the fewest that fit the shared memory; 0 if even 16 do not.
inline int sf_cluster(int64_t N, int D, int K) {
  if (N < 1 || D < 1 || K < 1 || (int64_t)N * D > (int64_t)kSfMaxCluster * 50000) return 0;
  int c0 = (int)std::min<int64_t>(kSfMaxCluster, std::max<int64_t>(1, (N + 639) / 640));
  for (int C = c0; C <= kSfMaxCluster; C++)
    if (sf_layout(N, D, K, C).total <= kSfMaxSmem) return C;
  return 0;
}

__device__ __forceinline__ double ld_cluster_f64(uint32_t addr) {
  double v;
  asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(addr) : "memory");
  return v;
}

// c_k and 1/var of the parameters in shared memory (one thread per component
// for c_k, all threads for 1/var).
__device__ __forceinline__ void sf_derive(int D, int K, const float* w, const float* var,
                                          float* iv, float* cst) {
  for (int i = threadIdx.x; i < K * D; i += blockDim.x) iv[i] = 1.0f / var[i];
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    double s = 0.0;
    for (int d = 0; d < D; d++) s += log(2.0 * M_PI * (double)var[(size_t)k * D + d]);
    cst[k] = w[k] > 0.f ? (float)(log((double)w[k]) - 0.5 * s) : -INFINITY;
  }
}

template <typename XT>
__global__ void __launch_bounds__(kSfThreads, 1)
    small_fit_kernel(const XT* __restrict__ X, int64_t N, int D, int K, int iters,
                     float var_floor, float* __restrict__ w_out, float* __restrict__ mu_out,
                     float* __restrict__ var_out, double* __restrict__ ll_hist,
                     unsigned int* status) {
  using namespace sm100;
  extern __shared__ __align__(16) uint8_t sm[];
  const int C = (int)cluster_nctarank();
  const uint32_t rank = cluster_ctarank();
  const SfLayout L = sf_layout(N, D, K, C);
  float* xs = reinterpret_cast<float*>(sm + L.x);
  float* rs = reinterpret_cast<float*>(sm + L.r);
  float* ws = reinterpret_cast<float*>(sm + L.w);
  float* mus = reinterpret_cast<float*>(sm + L.mu);
  float* vars = reinterpret_cast<float*>(sm + L.var);
  float* ivs = reinterpret_cast<float*>(sm + L.iv);
  float* cst = reinterpret_cast<float*>(sm + L.cst);
  double* part = reinterpret_cast<double*>(sm + L.part);
  double* tot = reinterpret_cast<double*>(sm + L.tot);
  double* red = reinterpret_cast<double*>(sm + L.red);
  const int tid = threadIdx.x;
  const size_t KD = (size_t)K * D;
  const uint32_t S = (uint32_t)K * (2u * D + 1u) + 1u;
  const int64_t r0 = (int64_t)rank * L.rows;
  const int nrows = (int)std::max<int64_t>(0, std::min<int64_t>(L.rows, N - r0));

  // this CTA's rows of X, and the starting parameters
  bool bad = false;
  for (int64_t i = tid; i < (int64_t)nrows * D; i += kSfThreads) {
    const float v = load1<XT>(X + (size_t)r0 * D, (int)i);
    if (!isfinite(v)) bad = true;
    const int64_t n = i / D;
    xs[(size_t)(i - n * D) * L.rows + n] = v;  // [d][n]
  }
  if (bad) atomicOr(status, GMM_DEVFLAG_NONFINITE_X);
  bool badp = false;
  for (int i = tid; i < K; i += kSfThreads) {
    ws[i] = w_out[i];
    if (!(ws[i] >= 0.f) || !isfinite(ws[i])) badp = true;
  }
  for (size_t i = tid; i < KD; i += kSfThreads) {
    mus[i] = mu_out[i];
    vars[i] = var_out[i];
    if (!isfinite(mus[i]) || !(vars[i] > 0.f) || !isfinite(vars[i])) badp = true;
  }
  if (badp && rank == 0) atomicOr(status, GMM_DEVFLAG_BAD_PARAMS);
  __syncthreads();
  sf_derive(D, K, ws, vars, ivs, cst);
  __syncthreads();

  for (int t = 0; t < iters; t++) {
    // 1. responsibilities of this CTA's rows
    double ll = 0.0;
    const size_t R = (size_t)L.rows;
    for (int n = tid; n < nrows; n += kSfThreads) {
      const float* x = xs + n;  // x[d * R]
      float* rr = rs + n;       // rr[k * R]
      float M = -INFINITY;
      for (int k = 0; k < K; k++) {
        float l = -INFINITY;
        if (cst[k] > -INFINITY) {
          const float* mk = mus + (size_t)k * D;
          const float* ik = ivs + (size_t)k * D;
          float q = 0.f;
          for (int d = 0; d < D; d++) {
            const float e = x[(size_t)d * R] - mk[d];
            q = fmaf(e * e, ik[d], q);
          }
          l = cst[k] - 0.5f * q;
        }
        rr[(size_t)k * R] = l;
        M = fmaxf(M, l);
      }
      float se = 0.f;
      for (int k = 0; k < K; k++)
        if (rr[(size_t)k * R] > -INFINITY) se += expf(rr[(size_t)k * R] - M);
      const float lse = M + logf(se);
      for (int k = 0; k < K; k++) {
        const float l = rr[(size_t)k * R];
        rr[(size_t)k * R] = l > -INFINITY ? expf(l - lse) : 0.f;
      }
      ll += (double)lse;
    }
    red[tid] = ll;
    __syncthreads();
    // 2. statistics about the iteration's input means, rows in order
    double* pb = part + (size_t)(t & 1) * S;
    for (size_t p = tid; p < KD; p += kSfThreads) {
      const int k = (int)(p / D), d = (int)(p - (size_t)k * D);
      const double m = (double)mus[p];
      double a = 0.0, b = 0.0;
      const float* rk = rs + (size_t)k * R;
      const float* xd = xs + (size_t)d * R;
      for (int n = 0; n < nrows; n++) {
        const double r = (double)rk[n];
        const double dx = (double)xd[n] - m;
        a += r * dx;
        b += r * dx * dx;
      }
      pb[K + p] = a;
      pb[K + KD + p] = b;
    }
    for (int k = tid; k < K; k += kSfThreads) {
      double nk = 0.0;
      for (int n = 0; n < nrows; n++) nk += (double)rs[(size_t)k * R + n];
      pb[k] = nk;
    }
    if (tid == 0) {
      double s = 0.0;
      for (int i = 0; i < kSfThreads; i++) s += red[i];  // thread order
      pb[S - 1] = s;
    }
    // 3. every CTA's partial is complete; sum them in CTA order, then the M-step
    cluster_sync();
    const uint32_t pb_addr = smem_u32(pb);
    for (uint32_t i = tid; i < S; i += kSfThreads) {
      double s = 0.0;
      for (int c = 0; c < C; c++) s += ld_cluster_f64(map_to_rank(pb_addr + 8u * i, (uint32_t)c));
      tot[i] = s;
    }
    __syncthreads();
    if (rank == 0 && tid == 0 && ll_hist) ll_hist[t] = tot[S - 1];
    for (size_t p = tid; p < KD; p += kSfThreads) {
      const int k = (int)(p / D);
      const double nk = tot[k];
      if (p - (size_t)k * D == 0) ws[k] = (float)(nk / (double)N);
      if (nk > 1e-12 * (double)N) {
        const double delta = tot[K + p] / nk;
        double v = tot[K + KD + p] / nk - delta * delta;
        if (!(v > (double)var_floor)) v = (double)var_floor;
        mus[p] = (float)((double)mus[p] + delta);
        vars[p] = (float)v;
      }
    }
    __syncthreads();
    sf_derive(D, K, ws, vars, ivs, cst);
    __syncthreads();
  }
  if (rank == 0) {
    for (int i = tid; i < K; i += kSfThreads) w_out[i] = ws[i];
    for (size_t i = tid; i < KD; i += kSfThreads) {
      mu_out[i] = mus[i];
      var_out[i] = vars[i];
    }
  }
  cluster_sync();  // no CTA leaves while another may still read its partials
}

}  // namespace scem
