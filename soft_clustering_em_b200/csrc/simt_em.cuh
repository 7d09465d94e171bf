// simt_em.cuh -- CUDA-core kernels of the fused EM step: parameter prep, the
// fused E-step + statistics pass for shapes the tensor-core kernel does not
// take, the deterministic reduction + M-step, top-m assignment and init.
//
// Method: "Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering"
// (review page, section 3): per data tile compute the E-step and the tile's
// sufficient statistics, accumulate them globally, never store N x K.
#pragma once

#include <math.h>

#include "common.cuh"

namespace scem {

// ---------------------------------------------------------------------------
// Parameter prep: one block per component.
//   pmu[d][k] = mu_kd, piv[d][k] = 1/var_kd (transposed for coalesced reads),
//   plogc[k]  = log pi_k - 1/2 sum_d log(2 pi var_kd), formed in fp64.
// Flags non-finite means, var <= 0 and w < 0 as GMM_DEVFLAG_BAD_PARAMS.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) prep_kernel(int D, int K, const float* __restrict__ w,
                                                   const float* __restrict__ mu,
                                                   const float* __restrict__ var, WsPtrs ws) {
  const int k = blockIdx.x;
  double s = 0.0;
  bool bad = false;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    const float m = mu[(size_t)k * D + d];
    const float v = var[(size_t)k * D + d];
    if (!isfinite(m) || !isfinite(v) || !(v > 0.f)) bad = true;
    ws.pmu[(size_t)d * K + k] = m;
    ws.piv[(size_t)d * K + k] = 1.0f / v;
    s += log(2.0 * M_PI * (double)v);
  }
  __shared__ double red[4];
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    const double S = red[0] + red[1] + red[2] + red[3];
    const float wk = w[k];
    if (!isfinite(wk) || !(wk >= 0.f)) bad = true;
    ws.plogc[k] = (wk > 0.f) ? (float)(log((double)wk) - 0.5 * S) : -INFINITY;
  }
  if (bad) atomicOr(ws.status, GMM_DEVFLAG_BAD_PARAMS);
}

// Logits of component k for the TN rows of the tile held in shared memory:
//   l_nk = plogc_k - 1/2 sum_d (x_nd - mu_kd)^2 / var_kd      (direct form)
// xs is TN x Dp (Dp = D rounded up to 4, zero padded); k >= K gives -inf.
template <int TN>
__device__ __forceinline__ void simt_logits(const float* __restrict__ xs, int Dp, int D, int K,
                                            int k, const WsPtrs& ws, float (&acc)[TN]) {
#pragma unroll
  for (int n = 0; n < TN; n++) acc[n] = 0.f;
  if (k >= K) {
#pragma unroll
    for (int n = 0; n < TN; n++) acc[n] = -INFINITY;
    return;
  }
  for (int d = 0; d < D; d += 4) {
    float m4[4], i4[4];
#pragma unroll
    for (int j = 0; j < 4; j++) {
      const bool ok = d + j < D;
      m4[j] = ok ? ws.pmu[(size_t)(d + j) * K + k] : 0.f;
      i4[j] = ok ? ws.piv[(size_t)(d + j) * K + k] : 0.f;
    }
#pragma unroll
    for (int n = 0; n < TN; n++) {
      const float4 x = *reinterpret_cast<const float4*>(xs + n * Dp + d);
      float e = x.x - m4[0];
      acc[n] = fmaf(e * e, i4[0], acc[n]);
      e = x.y - m4[1];
      acc[n] = fmaf(e * e, i4[1], acc[n]);
      e = x.z - m4[2];
      acc[n] = fmaf(e * e, i4[2], acc[n]);
      e = x.w - m4[3];
      acc[n] = fmaf(e * e, i4[3], acc[n]);
    }
  }
  const float c = ws.plogc[k];
#pragma unroll
  for (int n = 0; n < TN; n++) acc[n] = c - 0.5f * acc[n];
}

// (a, ai) ranks before (b, bi): larger value first, equal values by lower index.
__device__ __forceinline__ bool rank_before(float a, int ai, float b, int bi) {
  return a > b || (a == b && ai < bi);
}

enum SimtMode { kModeStats = 0, kModeLoglik = 1, kModeTopm = 2 };

// Shared-memory bytes of simt_fused_kernel for dimension D.
inline size_t simt_smem_bytes(int D) {
  const int Dp = (D + 3) & ~3;
  return sizeof(float) * ((size_t)kSimtRows * Dp + (size_t)kSimtRows * kSimtThreads +
                          3 * kSimtRows + 2 * kSimtRows * kMaxTopM);
}

// ---------------------------------------------------------------------------
// Fused pass over row tiles of kSimtRows points; CTA b takes tiles b, b+P, ...
// (static assignment: results do not depend on scheduling).
// Pass 1 over component chunks: logits -> online row max / sum-exp (and the
// running top-m in kModeTopm).  LSE_n = max + log(sum).
// Pass 2 (kModeStats): recompute the logits, r = exp(l - LSE), and add the
// tile's N_k, A = sum r (x - mu), B = sum r (x - mu)^2 into this CTA's fp64
// slot.  Components whose responsibilities in the tile are all exactly zero
// are skipped (adding zeros changes nothing).
// ---------------------------------------------------------------------------
template <typename XT, int MODE>
__global__ void __launch_bounds__(kSimtThreads) simt_fused_kernel(
    const XT* __restrict__ X, int64_t N, int D, int K, WsPtrs ws, int m,
    int32_t* __restrict__ idx_out, float* __restrict__ resp_out) {
  constexpr int TN = kSimtRows, CH = kSimtThreads, NW = CH / 32;
  extern __shared__ float4 smem4[];
  float* smem = reinterpret_cast<float*>(smem4);
  const int Dp = (D + 3) & ~3;
  float* xs = smem;
  float* lb = xs + TN * Dp;
  float* rowM = lb + TN * CH;
  float* rowS = rowM + TN;
  float* lse = rowS + TN;
  float* topv = lse + TN;
  int* topi = reinterpret_cast<int*>(topv + TN * kMaxTopM);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  double* slot = ws.slots + (size_t)blockIdx.x * ws.slot_stride;
  double* sN = slot;
  double* sA = slot + K;
  double* sB = sA + (size_t)K * D;
  double* sLL = sB + (size_t)K * D;
  if (MODE == kModeStats)
    for (size_t i = tid; i < ws.slot_stride; i += CH) slot[i] = 0.0;
  double ll = 0.0;

  const int64_t ntiles = (N + TN - 1) / TN;
  for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
    const int64_t row0 = t * TN;
    __syncthreads();
    bool bad = false;
    for (int i = tid; i < TN * Dp; i += CH) {
      const int n = i / Dp, d = i - n * Dp;
      float v = 0.f;
      if (d < D && row0 + n < N) {
        v = load_x(X, (size_t)(row0 + n) * D + d);
        if (!isfinite(v)) bad = true;
      }
      xs[i] = v;
    }
    if (bad) atomicOr(ws.status, GMM_DEVFLAG_NONFINITE_X);
    if (tid < TN) {
      rowM[tid] = -INFINITY;
      rowS[tid] = 0.f;
    }
    if (MODE == kModeTopm)
      for (int i = tid; i < TN * kMaxTopM; i += CH) {
        topv[i] = -INFINITY;
        topi[i] = 0x7fffffff;
      }
    __syncthreads();

    // ---- pass 1: row max / sum-exp (and top-m) over component chunks ----
    for (int c0 = 0; c0 < K; c0 += CH) {
      float acc[TN];
      simt_logits<TN>(xs, Dp, D, K, c0 + tid, ws, acc);
#pragma unroll
      for (int n = 0; n < TN; n++) lb[n * CH + tid] = acc[n];
      __syncthreads();
      for (int n = warp; n < TN; n += NW) {
        float v[CH / 32];
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < CH / 32; j++) {
          v[j] = lb[n * CH + lane + 32 * j];
          mx = fmaxf(mx, v[j]);
        }
        mx = warp_max(mx);
        const float Mold = rowM[n];
        const float Mnew = fmaxf(Mold, mx);
        if (Mnew > -INFINITY) {
          float s = 0.f;
#pragma unroll
          for (int j = 0; j < CH / 32; j++) s += expf(v[j] - Mnew);
          s = warp_sum(s);
          if (lane == 0) {
            rowS[n] = rowS[n] * expf(Mold - Mnew) + s;
            rowM[n] = Mnew;
          }
        }
        if (MODE == kModeTopm) {
          float rv = lane < m ? topv[n * kMaxTopM + lane] : -INFINITY;
          int ri = lane < m ? topi[n * kMaxTopM + lane] : 0x7fffffff;
          bool rtaken = lane >= m;
          unsigned taken = 0;
          float myv = -INFINITY;
          int myi = 0x7fffffff;
          for (int s = 0; s < m; s++) {
            float bv = -INFINITY;
            int bi = 0x7fffffff, bslot = -1;
            if (!rtaken && rank_before(rv, ri, bv, bi)) {
              bv = rv;
              bi = ri;
              bslot = CH / 32;
            }
#pragma unroll
            for (int j = 0; j < CH / 32; j++) {
              const int ci = c0 + lane + 32 * j;
              if (!((taken >> j) & 1u) && ci < K && rank_before(v[j], ci, bv, bi)) {
                bv = v[j];
                bi = ci;
                bslot = j;
              }
            }
            float wv = bv;
            int wi = bi;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              const float ov = __shfl_xor_sync(0xffffffffu, wv, o);
              const int oi = __shfl_xor_sync(0xffffffffu, wi, o);
              if (rank_before(ov, oi, wv, wi)) {
                wv = ov;
                wi = oi;
              }
            }
            if (bslot >= 0 && bi == wi) {
              if (bslot == CH / 32)
                rtaken = true;
              else
                taken |= 1u << bslot;
            }
            if (lane == s) {
              myv = wv;
              myi = wi;
            }
          }
          __syncwarp();
          if (lane < m) {
            topv[n * kMaxTopM + lane] = myv;
            topi[n * kMaxTopM + lane] = myi;
          }
        }
      }
      __syncthreads();
    }
    if (tid < TN) lse[tid] = rowM[tid] + logf(rowS[tid]);
    __syncthreads();
    if (tid == 0)
      for (int n = 0; n < TN && row0 + n < N; n++) ll += (double)lse[n];

    if (MODE == kModeTopm) {
      for (int n = warp; n < TN; n += NW) {
        const int64_t row = row0 + n;
        if (row < N && lane < m) {
          idx_out[row * m + lane] = topi[n * kMaxTopM + lane];
          resp_out[row * m + lane] = expf(topv[n * kMaxTopM + lane] - lse[n]);
        }
      }
    }

    // ---- pass 2: responsibilities and this tile's statistics ----
    if (MODE == kModeStats) {
      for (int c0 = 0; c0 < K; c0 += CH) {
        const int k = c0 + tid;
        if (k >= K) continue;
        float r[TN];
        simt_logits<TN>(xs, Dp, D, K, k, ws, r);
        float nk = 0.f;
#pragma unroll
        for (int n = 0; n < TN; n++) {
          r[n] = (row0 + n < N) ? expf(r[n] - lse[n]) : 0.f;
          nk += r[n];
        }
        if (nk == 0.f) continue;  // every responsibility of k in this tile is exactly 0
        sN[k] += (double)nk;
        for (int d = 0; d < D; d += 4) {
          float m4[4], a4[4] = {0.f, 0.f, 0.f, 0.f}, b4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int j = 0; j < 4; j++) m4[j] = (d + j < D) ? ws.pmu[(size_t)(d + j) * K + k] : 0.f;
#pragma unroll
          for (int n = 0; n < TN; n++) {
            const float4 x = *reinterpret_cast<const float4*>(xs + n * Dp + d);
            const float xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int j = 0; j < 4; j++) {
              const float e = xv[j] - m4[j];
              const float te = r[n] * e;
              a4[j] += te;
              b4[j] = fmaf(te, e, b4[j]);
            }
          }
#pragma unroll
          for (int j = 0; j < 4; j++)
            if (d + j < D) {
              sA[(size_t)(d + j) * K + k] += (double)a4[j];
              sB[(size_t)(d + j) * K + k] += (double)b4[j];
            }
        }
      }
    }
  }
  if (tid == 0 && MODE != kModeTopm) *sLL = ll;
}

// Fixed-order fp64 sum of the P slots into the canonical statistics buffer
// (component-major, moments about the means the step started from):
//   stats = [ N_k (K) | A (K x D) | B (K x D) | LL ].
__global__ void __launch_bounds__(256) simt_reduce_stats_kernel(int D, int K, WsPtrs ws,
                                                                double* __restrict__ stats) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t KD = (size_t)K * D;
  if (i == 0) {
    double ll = 0.0;
    for (int p = 0; p < ws.P; p++) ll += ws.slots[(size_t)p * ws.slot_stride + K + 2 * KD];
    stats[K + 2 * KD] = ll;
  }
  if (i >= KD) return;
  const int d = (int)(i / K), k = (int)(i - (size_t)d * K);
  double nk = 0.0, a = 0.0, b = 0.0;
  for (int p = 0; p < ws.P; p++) {
    const double* s = ws.slots + (size_t)p * ws.slot_stride;
    nk += s[k];
    a += s[K + i];
    b += s[K + KD + i];
  }
  if (d == 0) stats[k] = nk;
  stats[K + (size_t)k * D + d] = a;
  stats[K + KD + (size_t)k * D + d] = b;
}

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

// LL only: fixed-order sum of the per-CTA LL partials.
__global__ void reduce_loglik_kernel(int D, int K, WsPtrs ws, double* __restrict__ loglik) {
  double ll = 0.0;
  for (int p = 0; p < ws.P; p++)
    ll += ws.slots[(size_t)p * ws.slot_stride + (size_t)K * (2 * (size_t)D + 1)];
  *loglik = ll;
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
