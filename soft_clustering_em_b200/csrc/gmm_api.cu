// gmm_api.cu -- host side of the C ABI declared in include/gmm.h: argument
// checks, workspace layout and the launch sequence of each entry point.
// Nothing here allocates device memory or synchronises, except
// gmm_device_status.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <unordered_set>
#include <vector>

#include "common.cuh"
#include "gmm.h"
#include "ivf.cuh"
#include "mstep_init.cuh"
#include "small_fit.cuh"
#include "tc_em.cuh"
#include "tma_host.h"
#include "variants.cuh"

using namespace scem;

namespace {

size_t elem_bytes(int32_t t) { return t == GMM_BF16 ? 2 : 4; }

gmm_status check_problem(const gmm_problem* p) {
  if (!p) return GMM_ERR_INVALID_ARG;
  if (p->N < 1 || p->D < 1 || p->K < 1) return GMM_ERR_INVALID_ARG;
  if (p->xdtype != GMM_F32 && p->xdtype != GMM_BF16) return GMM_ERR_INVALID_ARG;
  if (!(p->var_floor >= 0.f) || !isfinite(p->var_floor)) return GMM_ERR_INVALID_ARG;
  if (p->D > kMaxD || p->K > kMaxK) return GMM_ERR_UNSUPPORTED;
  if ((size_t)p->N > ((size_t)1 << 40)) return GMM_ERR_UNSUPPORTED;
  return GMM_OK;
}

gmm_status check_x(const gmm_problem* p, const void* X) {
  if (!X) return GMM_ERR_INVALID_ARG;
  if (((uintptr_t)X) % 16 != 0) return GMM_ERR_UNSUPPORTED;
  if (((size_t)p->D * elem_bytes(p->xdtype)) % 16 != 0) return GMM_ERR_UNSUPPORTED;
  return GMM_OK;
}

gmm_status device_sms(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return GMM_ERR_CUDA;
  }
  if (cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return GMM_ERR_CUDA;
  }
  return GMM_OK;
}

// Where a problem's data sits in the workspace.  The init scratch always
// exists; the tensor-core layout exists when the shape has a tensor-core plan
// (every EM call needs one).  Both start at offset 256, after the shared
// status word, and the workspace covers the larger one.
struct Plan {
  InitLayout init;
  TcLayout tc;
  bool use_tc;
  size_t stats;  // canonical statistics buffer: K(2D+1)+1 doubles
  size_t aux;    // the variants' parameters: K x D variances, K weights, one shared variance
  size_t total;
};

size_t stats_doubles(const gmm_problem* p) { return (size_t)p->K * (2 * (size_t)p->D + 1) + 1; }

Plan make_plan(const gmm_problem* p, int sms, size_t cap) {
  Plan P;
  const size_t sbytes = align_up(stats_doubles(p) * 8, 256);
  // (less 256 bytes: the regions below start on 256-byte boundaries)
  const size_t c = cap ? (cap > sbytes + 256 ? cap - sbytes - 256 : 1) : 0;
  P.init = init_layout(p->D, p->K, sms);
  P.use_tc = tc_shape_ok(p->D, p->K, sms);
  if (P.use_tc) {
    P.tc = tc_layout(p->D, p->K, sms, c);
    if (P.tc.P < 1) P.use_tc = false;
  }
  size_t body = P.init.total;
  if (P.use_tc) body = std::max(body, P.tc.total);
  P.stats = align_up(body, 256);
  P.aux = P.stats + sbytes;
  P.total = P.aux + align_up(((size_t)p->K * p->D + p->K + 1) * 4, 256);
  return P;
}

gmm_status get_plan(const gmm_problem* p, void* ws, size_t ws_bytes, Plan* P) {
  int sms = 0;
  gmm_status s = device_sms(&sms);
  if (s != GMM_OK) return s;
  *P = make_plan(p, sms, 0);
  if (!ws || ((uintptr_t)ws) % 256 != 0 || ws_bytes < P->total) return GMM_ERR_WORKSPACE;
  return GMM_OK;
}

std::atomic<unsigned long long> g_launches{0};  // kernels enqueued by this library, all threads

gmm_status launch_status() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    fprintf(stderr, "gmm: CUDA launch failed: %s\n", cudaGetErrorString(e));
    return GMM_ERR_CUDA;
  }
  return GMM_OK;
}

std::atomic<cudaEvent_t> g_trace_start{nullptr}, g_trace_stop{nullptr};

void trace_begin(cudaStream_t st) {
  if (cudaEvent_t e = g_trace_start.load()) cudaEventRecord(e, st);
}
void trace_end(cudaStream_t st) {
  if (cudaEvent_t e = g_trace_stop.load()) cudaEventRecord(e, st);
}

// Status after enqueuing n kernels (counted for gmm_launch_count).
gmm_status launched(int n) {
  g_launches += n;
  return launch_status();
}

// One walk of gmm_ivf_build over all chunks, for m candidates per point.
template <int kM, bool kFill, bool kShared>
void ivf_walk_launch(int64_t N, int K, const int32_t* idx, const float* resp, float tau,
                     const IvfLayout& L, int64_t* cnt, const int64_t* offsets, int64_t* ids,
                     unsigned int* status, cudaStream_t st) {
  const int ctas = (L.B + kIvfWarps - 1) / kIvfWarps;
  const size_t smem = kShared ? (size_t)K * kIvfWarps * 4 : 0;
  auto kern = ivf_walk_kernel<kM, kFill, kShared>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess)
    return;  // the launch below fails and the caller's launch check reports it
  kern<<<ctas, kIvfWarps * 32, smem, st>>>(N, K, idx, resp, tau, L.B, L.R, cnt, offsets, ids,
                                           status);
}

template <int kM>
void ivf_walk_m(bool fill, int64_t N, int K, const int32_t* idx, const float* resp, float tau,
                const IvfLayout& L, int64_t* cnt, const int64_t* offsets, int64_t* ids,
                unsigned int* status, cudaStream_t st) {
  const bool sh = ivf_shared_counters(K, L.R, kM);
  if (fill && sh)
    ivf_walk_launch<kM, true, true>(N, K, idx, resp, tau, L, cnt, offsets, ids, status, st);
  else if (fill)
    ivf_walk_launch<kM, true, false>(N, K, idx, resp, tau, L, cnt, offsets, ids, status, st);
  else if (sh)
    ivf_walk_launch<kM, false, true>(N, K, idx, resp, tau, L, cnt, offsets, ids, status, st);
  else
    ivf_walk_launch<kM, false, false>(N, K, idx, resp, tau, L, cnt, offsets, ids, status, st);
}

void ivf_walk(int m, bool fill, int64_t N, int K, const int32_t* idx, const float* resp,
              float tau, const IvfLayout& L, int64_t* cnt, const int64_t* offsets, int64_t* ids,
              unsigned int* status, cudaStream_t st) {
  switch (m) {
    case 1: return ivf_walk_m<1>(fill, N, K, idx, resp, tau, L, cnt, offsets, ids, status, st);
    case 2: return ivf_walk_m<2>(fill, N, K, idx, resp, tau, L, cnt, offsets, ids, status, st);
    case 3: return ivf_walk_m<3>(fill, N, K, idx, resp, tau, L, cnt, offsets, ids, status, st);
    case 4: return ivf_walk_m<4>(fill, N, K, idx, resp, tau, L, cnt, offsets, ids, status, st);
    case 5: return ivf_walk_m<5>(fill, N, K, idx, resp, tau, L, cnt, offsets, ids, status, st);
    case 6: return ivf_walk_m<6>(fill, N, K, idx, resp, tau, L, cnt, offsets, ids, status, st);
    case 7: return ivf_walk_m<7>(fill, N, K, idx, resp, tau, L, cnt, offsets, ids, status, st);
    default: return ivf_walk_m<8>(fill, N, K, idx, resp, tau, L, cnt, offsets, ids, status, st);
  }
}

// ---------------------------------------------------------------------------
// Tensor-core path
// ---------------------------------------------------------------------------
constexpr uint64_t kWaitBudgetNs = 1000000000ull;  // default: 1 s per device-side wait
std::atomic<uint64_t> g_wait_budget_ns{kWaitBudgetNs};  // gmm_set_wait_budget

gmm_status tc_prep(const gmm_problem* p, const float* w, const float* mu, const float* var,
                   char* ws, const TcLayout& T, cudaStream_t st) {
  float* m = (float*)(ws + T.m);
  tc_center_kernel<<<p->D, 256, 0, st>>>(p->D, p->K, w, mu, var, m,
                                                       (float*)(ws + T.isc), (float*)(ws + T.sc));
  const size_t psmem = tc_prep_smem_bytes(p->D, T.Fpad);
  // (set every time: the static shared memory adds to the dynamic size)
  if (cudaFuncSetAttribute(tc_prep_w_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)psmem) != cudaSuccess) {
    cudaGetLastError();
    return GMM_ERR_UNSUPPORTED;
  }
  tc_prep_w_kernel<<<T.Kpad, 128, psmem, st>>>(
      p->N, p->D, p->K, T.Fpad, w, mu, var, m, (const float*)(ws + T.sc), (__half*)(ws + T.whi),
      (__half*)(ws + T.wlo), (float*)(ws + T.c), (float*)(ws + T.wsc), (int*)(ws + T.ndir),
      (int*)(ws + T.nsplit), (float*)(ws + T.muh), (float*)(ws + T.ph), (int*)(ws + T.precise),
      (float*)(ws + T.ci), (float*)(ws + T.cx), (float*)(ws + T.mg), (uint16_t*)(ws + T.perm),
      (float*)(ws + T.mun), (float*)(ws + T.pn),
      (uint32_t*)(ws + T.pmask), (uint16_t*)(ws + T.rank), (unsigned long long*)(ws + T.dirq),
      (unsigned int*)ws);
  return launched(2);
}

// Clusters of the fused pass: as many as fit at once, at most one per slot
// (and, with one group, no more than there are tiles); with G > 1 groups a
// whole number per group, the same for every chunk of a step.
template <typename XT, int MODE, int FSRC>
gmm_status tc_clusters(const TcLayout& T, int64_t ntiles, size_t smem, int* ncl_out) {
  auto kern = tc_fused_kernel<XT, MODE, FSRC>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess) {
    cudaGetLastError();
    return GMM_ERR_UNSUPPORTED;
  }
  if (T.C > 8 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    return GMM_ERR_UNSUPPORTED;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)T.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.blockDim = dim3(kTcThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.gridDim = dim3((unsigned)(T.C * T.P), 1, 1);
  int max_clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&max_clusters, (void*)kern, &cfg) != cudaSuccess ||
      max_clusters < 1) {
    cudaGetLastError();
    return GMM_ERR_UNSUPPORTED;
  }
  int ncl = std::min(T.P, max_clusters);
  if (T.G == 1)
    ncl = (int)std::min<int64_t>(ncl, ntiles);
  else
    ncl = ncl / T.G * T.G;
  if (ncl < 1) return GMM_ERR_UNSUPPORTED;
  *ncl_out = ncl;
  return GMM_OK;
}

// One launch of the fused kernel over rows [0, N) of X with ncl clusters.
// FSRC = 1: the rows' features are in the workspace's chunk buffer.
template <typename XT, int MODE, int FSRC>
gmm_status tc_launch(const gmm_problem* p, const void* X, int64_t N, char* ws, const TcLayout& T,
                     int ncl, int accumulate, cudaStream_t st, int32_t* labels = nullptr,
                     int ncand = 0, int fg0 = 0, int nfgc = 0, int rmode = 0) {
  CUtensorMap mhi, mlo, fhi, flo;
  memset(&mhi, 0, sizeof(mhi));
  memset(&mlo, 0, sizeof(mlo));
  memset(&fhi, 0, sizeof(fhi));
  memset(&flo, 0, sizeof(flo));
  if (!make_tmap_16b_sw128(&mhi, ws + T.whi, (uint64_t)T.Fpad, (uint64_t)T.Kpad,
                            (uint64_t)T.Fpad * 2, kTcComps) ||
      !make_tmap_16b_sw128(&mlo, ws + T.wlo, (uint64_t)T.Fpad, (uint64_t)T.Kpad,
                            (uint64_t)T.Fpad * 2, kTcComps))
    return GMM_ERR_CUDA;
  if (FSRC && (!make_tmap_16b_sw128(&fhi, ws + T.fhi, (uint64_t)T.Fpad, (uint64_t)N,
                                     (uint64_t)T.Fpad * 2, kTcRows) ||
               !make_tmap_16b_sw128(&flo, ws + T.flo, (uint64_t)T.Fpad, (uint64_t)N,
                                     (uint64_t)T.Fpad * 2, kTcRows)))
    return GMM_ERR_CUDA;
  const TcSmem S = tc_smem_layout(p->D, T.C, T.nchunks);
  // at least 120 KB so that exactly one CTA (and one 512-column TMEM allocation) sits on an SM
  const size_t smem = std::max<size_t>(S.total, 120 * 1024);
  auto kern = tc_fused_kernel<XT, MODE, FSRC>;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)T.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.blockDim = dim3(kTcThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.gridDim = dim3((unsigned)(T.C * ncl), 1, 1);
  TcArgs args;
  args.X = X;
  args.N = N;
  args.D = p->D;
  args.K = p->K;
  args.C = T.C;
  args.nchunks = T.nchunks;
  args.m = (const float*)(ws + T.m);
  args.isc = (const float*)(ws + T.isc);
  args.c = (const float*)(ws + T.c);
  args.ci = (const float*)(ws + T.ci);
  args.wsc = (const float*)(ws + T.wsc);
  args.ndir = (const int*)(ws + T.ndir);
  args.nsplit = (const int*)(ws + T.nsplit);
  args.muh = (const float*)(ws + T.muh);
  args.ph = (const float*)(ws + T.ph);
  args.perm = (const uint16_t*)(ws + T.perm);
  args.mun = (const float*)(ws + T.mun);
  args.pn = (const float*)(ws + T.pn);
  args.cx = (const float*)(ws + T.cx);
  args.mg = (const float*)(ws + T.mg);
  args.slots = (double*)(ws + T.slots);
  args.slot_stride = T.slot_stride;
  args.dirq = (unsigned long long*)(ws + T.dirq);
  args.Kpad = T.Kpad;
  args.G = T.G;
  args.part = (float2*)(ws + T.part);
  args.accumulate = accumulate;
  args.labels = labels;
  args.cand = (float2*)(ws + T.cand);
  args.rowst = (float2*)(ws + T.rowst);
  args.ncand = std::min(kTcCand, ncand);
  args.fg0 = fg0;
  args.nfgc = nfgc > 0 ? nfgc : T.nfg;
  args.nfg = T.nfg;
  args.rbuf = (uint8_t*)(ws + T.rbuf);
  args.rmode = rmode;
  args.status = (unsigned int*)ws;
  args.drain_tiles = kTcDrainTiles;
  args.precise = (const int*)(ws + T.precise);
  args.pmask = (const uint32_t*)(ws + T.pmask);
  args.wait_ns = g_wait_budget_ns.load();
  args.drain_ns = kWaitBudgetNs;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args, mhi, mlo, fhi, flo);
  if (e != cudaSuccess) {
    fprintf(stderr, "gmm: tensor-core launch failed: %s\n", cudaGetErrorString(e));
    cudaGetLastError();
    return GMM_ERR_CUDA;
  }
  return launched(1);
}

size_t tc_smem_bytes(const gmm_problem* p, const TcLayout& T) {
  return std::max<size_t>(tc_smem_layout(p->D, T.C, T.nchunks).total, 120 * 1024);
}

// Converts rows [r0, r0 + n) of X into the chunk's feature buffer.
template <typename XT>
gmm_status tc_convert(const gmm_problem* p, const XT* Xc, int64_t n, char* ws, const TcLayout& T,
                      cudaStream_t st) {
  const int64_t items = n * (p->D / 4);
  const unsigned grid = (unsigned)std::min<int64_t>((items + 255) / 256, 148 * 16);
  tc_convert_kernel<XT><<<grid, 256, 0, st>>>(Xc, n, p->D, T.Fpad, (const float*)(ws + T.m),
                                             (const float*)(ws + T.isc), (__half*)(ws + T.fhi),
                                             (__half*)(ws + T.flo), (unsigned int*)ws);
  return launched(1);
}

// The fused pass over pre-converted features (FS = 1: resident per tile;
// FS = 2: streamed in rounds), chunk by chunk: the features converted, the
// partial pass when there are several component groups, then the statistics
// pass once per feature group (or the log-likelihood).
template <typename XT, int MODE, int FS>
gmm_status tc_pass_chunked(const gmm_problem* p, const void* X, char* ws, const TcLayout& T,
                           cudaStream_t st, int* nslots, double* loglik, int32_t* labels) {
  constexpr int PART = tc_mode_hard(MODE) ? kTcHardPartial : kTcPartial;
  const int64_t ntiles = (p->N + kTcRows - 1) / kTcRows;
  const size_t smem = tc_smem_bytes(p, T);
  gmm_status s;
  int ncl = 1 << 30, c2 = 0;
  if (T.G > 1) {
    if ((s = tc_clusters<XT, PART, FS>(T, ntiles, smem, &c2)) != GMM_OK) return s;
    ncl = std::min(ncl, c2);
  }
  if ((s = tc_clusters<XT, MODE, FS>(T, ntiles, smem, &c2)) != GMM_OK) return s;
  ncl = std::min(ncl, c2);
  const size_t row_bytes = (size_t)p->D * sizeof(XT);
  double* blocks = (double*)(ws + T.slots);  // log-likelihood mode with groups: the slots are free
  trace_begin(st);
  int64_t i = 0;
  for (int64_t r0 = 0; r0 < p->N; r0 += T.R, i++) {
    const int64_t n = std::min<int64_t>(T.R, p->N - r0);
    const XT* Xc = (const XT*)((const char*)X + (size_t)r0 * row_bytes);
    if ((s = tc_convert<XT>(p, Xc, n, ws, T, st)) != GMM_OK) return s;
    if (T.G > 1 && (s = tc_launch<XT, PART, FS>(p, Xc, n, ws, T, ncl, 0, st)) != GMM_OK)
      return s;
    if (tc_mode_stats(MODE)) {
      // several feature groups: the first pass stores r^, the others load it
      for (int fg = 0; fg < T.NFG; fg++) {
        const int fg0 = fg * T.nfg;
        const int rmode = T.NFG == 1 ? 0 : fg == 0 ? 1 : 2;
        if ((s = tc_launch<XT, MODE, FS>(p, Xc, n, ws, T, ncl, !(i == 0 && fg == 0), st,
                                         labels ? labels + r0 : nullptr, 0, fg0,
                                         std::min(T.nfg, T.nchunks - fg0), rmode)) != GMM_OK)
          return s;
      }
    } else if (T.G > 1) {
      tc_part_loglik_kernel<<<kTcLseBlocks, 256, 0, st>>>((const float2*)(ws + T.part), n, T.G,
                                                          blocks);
      tc_sum_blocks_kernel<<<1, 1, 0, st>>>(blocks, i == 0, loglik);
      if ((s = launched(2)) != GMM_OK) return s;
    } else if ((s = tc_launch<XT, MODE, FS>(p, Xc, n, ws, T, ncl, i > 0, st)) != GMM_OK) {
      return s;  // one group, streamed features: each chunk's LL adds into the slots
    }
  }
  trace_end(st);
  *nslots = ncl;
  return GMM_OK;
}

// The fused pass over all rows of X: one launch with one component group and
// resident features; otherwise chunk by chunk (tc_pass_chunked).  *nslots
// receives the number of slots written.  The trace events bracket the pass.
template <typename XT, int MODE>
gmm_status tc_pass_t(const gmm_problem* p, const void* X, char* ws, const TcLayout& T,
                     cudaStream_t st, int* nslots, double* loglik, int32_t* labels) {
  if (tc_streamed(T.nchunks))
    return tc_pass_chunked<XT, MODE, 2>(p, X, ws, T, st, nslots, loglik, labels);
  if (T.G > 1) return tc_pass_chunked<XT, MODE, 1>(p, X, ws, T, st, nslots, loglik, labels);
  const int64_t ntiles = (p->N + kTcRows - 1) / kTcRows;
  gmm_status s;
  int ncl = 0;
  if ((s = tc_clusters<XT, MODE, 0>(T, ntiles, tc_smem_bytes(p, T), &ncl)) != GMM_OK) return s;
  trace_begin(st);
  s = tc_launch<XT, MODE, 0>(p, X, p->N, ws, T, ncl, 0, st, labels);
  trace_end(st);
  *nslots = ncl;
  return s;
}

template <int MODE>
gmm_status tc_pass(const gmm_problem* p, const void* X, char* ws, const TcLayout& T,
                   cudaStream_t st, int* nslots, double* loglik = nullptr,
                   int32_t* labels = nullptr) {
  if (p->xdtype == GMM_BF16)
    return tc_pass_t<__nv_bfloat16, MODE>(p, X, ws, T, st, nslots, loglik, labels);
  return tc_pass_t<float, MODE>(p, X, ws, T, st, nslots, loglik, labels);
}

// E-step and statistics of the rows of X into the canonical buffer `stats`.
// n_prep is the point count the tensor-core prep sizes its small-component
// rule by (pi_k * n_prep points): p->N, or the whole data's N when X is one
// chunk of it.
gmm_status estep_stats_impl(const gmm_problem* p, const void* X, const float* w,
                            const float* mu, const float* var, double* stats, void* ws_base,
                            const Plan& P, cudaStream_t st, int64_t n_prep,
                            bool hard = false, int32_t* labels = nullptr) {
  char* ws = (char*)ws_base;
  gmm_status s;
  const size_t KD = (size_t)p->K * p->D;
  const unsigned blocks = (unsigned)((KD + 255) / 256);
  if (!P.use_tc) return GMM_ERR_UNSUPPORTED;  // no tensor-core plan for this shape
  {
    const TcLayout& T = P.tc;
    gmm_problem pp = *p;
    pp.N = n_prep;
    if ((s = tc_prep(&pp, w, mu, var, ws, T, st)) != GMM_OK) return s;
    int nslots = 0;
    s = hard ? tc_pass<kTcHardStats>(p, X, ws, T, st, &nslots, nullptr, labels)
             : tc_pass<kTcStats>(p, X, ws, T, st, &nslots);
    if (s != GMM_OK) return s;
    tc_reduce_stats_kernel<<<blocks, 256, 0, st>>>(
        p->D, p->K, T.Kpad, (const float*)(ws + T.m), (const float*)(ws + T.sc), mu,
        (const uint16_t*)(ws + T.rank), (const int*)(ws + T.ndir), (const float*)(ws + T.ph),
        (const unsigned long long*)(ws + T.dirq), (const double*)(ws + T.slots), T.slot_stride,
        nslots, T.G, T.C * kTcComps, stats);
    return launched(1);
  }
}

// One chunk of the top-m pass over pre-converted features (FS = 1 or 2).
template <typename XT, int FS>
gmm_status tc_topm_chunk(const gmm_problem* p, const XT* Xc, int64_t n, char* ws,
                         const TcLayout& T, int nc, cudaStream_t st) {
  const int64_t ntiles = (n + kTcRows - 1) / kTcRows;
  const size_t smem = tc_smem_bytes(p, T);
  gmm_status s;
  int ncl = 1 << 30, c2 = 0;
  if (T.G > 1) {
    if ((s = tc_clusters<XT, kTcPartial, FS>(T, ntiles, smem, &c2)) != GMM_OK) return s;
    ncl = c2;
  }
  if ((s = tc_clusters<XT, kTcTopm, FS>(T, ntiles, smem, &c2)) != GMM_OK) return s;
  ncl = std::min(ncl, c2);
  if ((s = tc_convert<XT>(p, Xc, n, ws, T, st)) != GMM_OK) return s;
  if (T.G > 1 && (s = tc_launch<XT, kTcPartial, FS>(p, Xc, n, ws, T, ncl, 0, st)) != GMM_OK)
    return s;
  return tc_launch<XT, kTcTopm, FS>(p, Xc, n, ws, T, ncl, 0, st, nullptr, nc);
}

// Top-m assignment on the tensor cores, chunk by chunk (Rt rows): the top-m
// pass (after the features are converted and the partial pass, when the
// shape needs them) writes each (CTA, column half)'s candidates and each
// row's (max, sum-exp); tc_topm_refine_kernel finishes the rows in direct form.
template <typename XT>
gmm_status tc_topm_t(const gmm_problem* p, const void* X, const float* w, const float* mu,
                     const float* var, int m, int32_t* idx, float* resp, char* ws, const Plan& P,
                     cudaStream_t st) {
  const TcLayout& T = P.tc;
  gmm_status s;
  if ((s = tc_prep(p, w, mu, var, ws, T, st)) != GMM_OK) return s;
  float* iv = (float*)(ws + P.aux);
  float* c0 = iv + (size_t)p->K * p->D;
  tc_topm_prep_kernel<<<p->K, 128, 0, st>>>(p->D, w, var, iv, c0);
  if ((s = launched(1)) != GMM_OK) return s;
  const int nc = std::min(m + 2, kTcCand);
  const size_t smem = tc_smem_bytes(p, T);
  const size_t row_bytes = (size_t)p->D * sizeof(XT);
  const bool streamed = tc_streamed(T.nchunks);
  trace_begin(st);
  for (int64_t r0 = 0; r0 < p->N; r0 += T.Rt) {
    const int64_t n = std::min<int64_t>(T.Rt, p->N - r0);
    const XT* Xc = (const XT*)((const char*)X + (size_t)r0 * row_bytes);
    if (streamed) {
      s = tc_topm_chunk<XT, 2>(p, Xc, n, ws, T, nc, st);
    } else if (T.G > 1) {
      s = tc_topm_chunk<XT, 1>(p, Xc, n, ws, T, nc, st);
    } else {
      int ncl = 0;
      s = tc_clusters<XT, kTcTopm, 0>(T, (n + kTcRows - 1) / kTcRows, smem, &ncl);
      if (s == GMM_OK) s = tc_launch<XT, kTcTopm, 0>(p, Xc, n, ws, T, ncl, 0, st, nullptr, nc);
    }
    if (s != GMM_OK) return s;
    tc_topm_refine_kernel<XT><<<(unsigned)((n + 127) / 128), 128, 0, st>>>(
        Xc, n, p->D, p->K, T.G * T.C * 2, nc, m, (const float2*)(ws + T.cand),
        (const float2*)(ws + T.rowst), mu, iv, c0, idx + (size_t)r0 * m, resp + (size_t)r0 * m);
    if ((s = launched(1)) != GMM_OK) return s;
  }
  trace_end(st);
  return GMM_OK;
}

gmm_status mstep_impl(const gmm_problem* p, const double* stats, int nshards, float* w,
                      float* mu, float* var, double* loglik, cudaStream_t st) {
  const size_t KD = (size_t)p->K * p->D;
  mstep_kernel<<<(unsigned)((KD + 255) / 256), 256, 0, st>>>(p->N, p->D, p->K, p->var_floor,
                                                             stats, nshards, w, mu, var, loglik);
  return launched(1);
}

// total[i] += part[i]: one chunk's statistics into the running total (chunk order).
__global__ void __launch_bounds__(256) stats_add_kernel(double* __restrict__ total,
                                                        const double* __restrict__ part, size_t n) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) total[i] += part[i];
}

// Device staging of gmm_em_step_host: two chunk buffers, then the running and
// the per-chunk statistics.
struct HostStaging {
  size_t buf_bytes, stats_bytes, total;
};

HostStaging host_staging(const gmm_problem* p, int64_t chunk_rows) {
  HostStaging H;
  H.buf_bytes = align_up((size_t)chunk_rows * p->D * elem_bytes(p->xdtype), 256);
  H.stats_bytes = align_up(stats_doubles(p) * 8, 256);
  H.total = 2 * H.buf_bytes + 2 * H.stats_bytes;
  return H;
}

// Events of one gmm_em_step_host call, destroyed on every way out (a pending
// event is released once the work it marks has completed).
struct StagingEvents {
  cudaEvent_t copied[2] = {nullptr, nullptr}, used[2] = {nullptr, nullptr};
  bool create() {
    for (int b = 0; b < 2; ++b)
      if (cudaEventCreateWithFlags(&copied[b], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&used[b], cudaEventDisableTiming) != cudaSuccess)
        return false;
    return true;
  }
  ~StagingEvents() {
    for (int b = 0; b < 2; ++b) {
      if (copied[b]) cudaEventDestroy(copied[b]);
      if (used[b]) cudaEventDestroy(used[b]);
    }
  }
};

gmm_status em_step_impl(const gmm_problem* p, const void* X, float* w, float* mu, float* var,
                        double* loglik, void* ws_base, const Plan& P, cudaStream_t st) {
  double* stats = (double*)((char*)ws_base + P.stats);
  gmm_status s = estep_stats_impl(p, X, w, mu, var, stats, ws_base, P, st, p->N);
  if (s != GMM_OK) return s;
  return mstep_impl(p, stats, 1, w, mu, var, loglik, st);
}

// All iterations of a small fit in one launch of one cluster (small_fit.cuh).
// GMM_ERR_UNSUPPORTED when the cluster cannot be placed on this device.
template <typename XT>
gmm_status small_fit_t(const gmm_problem* p, const void* X, int iters, float* w, float* mu,
                       float* var, double* ll, unsigned int* status, cudaStream_t st) {
  const int C = sf_cluster(p->N, p->D, p->K);
  const size_t smem = sf_layout(p->N, p->D, p->K, C).total;
  auto kern = small_fit_kernel<XT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess ||
      (C > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                    cudaSuccess)) {
    cudaGetLastError();
    return GMM_ERR_UNSUPPORTED;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.blockDim = dim3(kSfThreads, 1, 1);
  cfg.gridDim = dim3((unsigned)C, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  int max_clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&max_clusters, (void*)kern, &cfg) != cudaSuccess ||
      max_clusters < 1) {
    cudaGetLastError();
    return GMM_ERR_UNSUPPORTED;
  }
  trace_begin(st);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, (const XT*)X, p->N, p->D, p->K, iters,
                                           p->var_floor, w, mu, var, ll, status);
  trace_end(st);
  if (e != cudaSuccess) {
    fprintf(stderr, "gmm: small-fit launch failed: %s\n", cudaGetErrorString(e));
    cudaGetLastError();
    return GMM_ERR_CUDA;
  }
  return launched(1);
}

gmm_status small_fit(const gmm_problem* p, const void* X, int iters, float* w, float* mu,
                     float* var, double* ll, unsigned int* status, cudaStream_t st) {
  if (p->xdtype == GMM_BF16)
    return small_fit_t<__nv_bfloat16>(p, X, iters, w, mu, var, ll, status, st);
  return small_fit_t<float>(p, X, iters, w, mu, var, ll, status, st);
}

// ---------------------------------------------------------------------------
// Scratch for gmm_em_step_noalloc: a fixed array in the module's own device
// memory, so that entry point never asks for memory.  It exists on every
// device that loads this library, for the life of the process.  Host code only
// sees a host-side stand-in under this name; the device address comes from
// cudaGetSymbolAddress, looked up once per device and cached.
// ---------------------------------------------------------------------------
constexpr size_t kNoallocScratchBytes = (size_t)32 << 20;
constexpr int kNoallocMaxDevices = 64;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];
std::mutex g_noalloc_mu;
// The address is looked up once per device and context: the context that was
// current at the lookup is kept beside it, and a call made under another one
// (a context created after cudaDeviceReset, or a non-primary driver context)
// looks the address up again.
struct NoallocEntry {
  void* ctx;
  void* ptr;
};
NoallocEntry g_noalloc_cache[kNoallocMaxDevices] = {};

typedef int (*CtxGetCurrentFn)(void**);

// The calling thread's current driver context (null if none or unknown),
// fetched through the runtime so the library does not link libcuda.
void* current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
    else
      cudaGetLastError();
    tried = true;
  }
  void* ctx = nullptr;
  if (!fn || fn(&ctx) != 0) return nullptr;
  return ctx;
}

gmm_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return GMM_ERR_CUDA;
  }
  if (dev < 0 || dev >= kNoallocMaxDevices) return GMM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  void* ctx = current_context();
  NoallocEntry& e = g_noalloc_cache[dev];
  if (!e.ptr || !ctx || e.ctx != ctx) {
    void* ptr = nullptr;
    const cudaError_t r = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (r != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return GMM_ERR_CUDA;
    }
    e.ctx = ctx;
    e.ptr = ptr;
  }
  *out = e.ptr;
  return GMM_OK;
}


// SplitMix64 in counter form (Steele, Lea and Flood, "Fast splittable
// pseudorandom number generators", OOPSLA 2014): the i-th output (i = 0, 1, ...)
// of the generator started from state `seed`.
uint64_t splitmix64_at(uint64_t seed, uint64_t i) {
  uint64_t z = seed + (i + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Uniform integer in [0, n) from the stream's next outputs (*ctr counts the
// outputs used): an output x is taken as x mod n when it lies below the
// largest multiple of n that fits in 64 bits, otherwise the next one is drawn,
// so every value is equally likely.
uint64_t uniform_below(uint64_t seed, uint64_t* ctr, uint64_t n) {
  const uint64_t rem = (0 - n) % n;  // 2^64 mod n
  for (;;) {
    const uint64_t x = splitmix64_at(seed, (*ctr)++);
    if (x <= ~rem) return x % n;  // x < 2^64 - rem
  }
}

// K distinct indices from [0, N), every K-subset equally likely: Floyd's
// algorithm (Bentley and Floyd, "A sample of brilliance", Programming Pearls,
// CACM 1987).  For j = N-K .. N-1 draw t uniform in [0, j]; take t, or j when t
// was already taken.  rows[k] is the index taken at step k.
void sample_rows(int64_t N, int K, uint64_t seed, std::vector<int64_t>* rows) {
  rows->clear();
  rows->reserve(K);
  std::unordered_set<int64_t> taken;
  taken.reserve(2 * (size_t)K);
  uint64_t ctr = 0;
  for (int64_t j = N - K; j < N; j++) {
    const int64_t t = (int64_t)uniform_below(seed, &ctr, (uint64_t)j + 1);
    const int64_t v = taken.count(t) ? j : t;
    taken.insert(v);
    rows->push_back(v);
  }
}

}  // namespace

extern "C" {

const char* gmm_status_string(gmm_status s) {
  switch (s) {
    case GMM_OK: return "GMM_OK";
    case GMM_ERR_INVALID_ARG: return "GMM_ERR_INVALID_ARG";
    case GMM_ERR_UNSUPPORTED: return "GMM_ERR_UNSUPPORTED";
    case GMM_ERR_CUDA: return "GMM_ERR_CUDA";
    case GMM_ERR_NUMERIC: return "GMM_ERR_NUMERIC";
    case GMM_ERR_TIMEOUT: return "GMM_ERR_TIMEOUT";
    case GMM_ERR_WORKSPACE: return "GMM_ERR_WORKSPACE";
  }
  return "GMM_ERR_UNKNOWN";
}

gmm_status gmm_workspace_size(const gmm_problem* p, size_t* bytes) {
  gmm_status s = check_problem(p);
  if (s != GMM_OK) return s;
  if (!bytes) return GMM_ERR_INVALID_ARG;
  int sms = 0;
  s = device_sms(&sms);
  if (s != GMM_OK) return s;
  *bytes = make_plan(p, sms, 0).total;
  return GMM_OK;
}

gmm_status gmm_init_rows(const gmm_problem* p, const void* X, const int64_t* rows_host,
                         int32_t init_var, float* w, float* mu, float* var, void* ws,
                         size_t ws_bytes, void* stream) {
  gmm_status s = check_problem(p);
  if (s != GMM_OK) return s;
  if ((s = check_x(p, X)) != GMM_OK) return s;
  if (!rows_host || !w || !mu || !var) return GMM_ERR_INVALID_ARG;
  if (init_var != GMM_INIT_VAR_ONE && init_var != GMM_INIT_VAR_DATA) return GMM_ERR_INVALID_ARG;
  for (int k = 0; k < p->K; k++)
    if (rows_host[k] < 0 || rows_host[k] >= p->N) return GMM_ERR_INVALID_ARG;
  Plan P;
  if ((s = get_plan(p, ws, ws_bytes, &P)) != GMM_OK) return s;
  int64_t* rows = (int64_t*)((char*)ws + P.init.rows);
  double* part = (double*)((char*)ws + P.init.part);
  const int nparts = P.init.P;
  cudaStream_t st = (cudaStream_t)stream;
  // the K row indices travel to the workspace (the one host->device copy of this call)
  if (cudaMemcpyAsync(rows, rows_host, sizeof(int64_t) * p->K, cudaMemcpyHostToDevice, st) !=
      cudaSuccess) {
    launch_status();
    return GMM_ERR_CUDA;
  }
  const bool bf = p->xdtype == GMM_BF16;
  if (bf)
    init_gather_kernel<__nv_bfloat16><<<p->K, 128, 0, st>>>((const __nv_bfloat16*)X, p->D, p->K,
                                                           rows, init_var, w, mu, var);
  else
    init_gather_kernel<float><<<p->K, 128, 0, st>>>((const float*)X, p->D, p->K, rows, init_var,
                                                    w, mu, var);
  if ((s = launched(1)) != GMM_OK) return s;
  if (init_var == GMM_INIT_VAR_DATA) {
    double* mean = part + (size_t)nparts * p->D;
    for (int pass = 0; pass < 2; pass++) {
      const double* mptr = pass == 0 ? nullptr : mean;
      if (bf)
        col_partial_kernel<__nv_bfloat16><<<nparts, 256, 0, st>>>((const __nv_bfloat16*)X, p->N,
                                                                  p->D, mptr, part);
      else
        col_partial_kernel<float><<<nparts, 256, 0, st>>>((const float*)X, p->N, p->D, mptr,
                                                          part);
      col_finish_kernel<<<(p->D + 127) / 128, 128, 0, st>>>(p->N, p->D, p->K, nparts, part, pass,
                                                            p->var_floor, mean, var);
      if ((s = launched(2)) != GMM_OK) return s;
    }
  }
  return GMM_OK;
}

gmm_status gmm_plan(const gmm_problem* p, gmm_plan_info* info) {
  gmm_status s = check_problem(p);
  if (s != GMM_OK) return s;
  if (!info) return GMM_ERR_INVALID_ARG;
  int sms = 0;
  if ((s = device_sms(&sms)) != GMM_OK) return s;
  const Plan P = make_plan(p, sms, 0);
  memset(info, 0, sizeof(*info));
  info->tensor_cores = P.use_tc ? 1 : 0;
  info->fit_one_launch = sf_cluster(p->N, p->D, p->K) > 0 ? 1 : 0;
  if (P.use_tc) {
    info->cluster_ctas = P.tc.C;
    info->groups = P.tc.G;
    info->chunk_rows = P.tc.G > 1 ? P.tc.R : 0;
  }
  return GMM_OK;
}

gmm_status gmm_init(const gmm_problem* p, const void* X, uint64_t seed, int32_t init_var,
                    float* w, float* mu, float* var, void* ws, size_t ws_bytes, void* stream) {
  gmm_status s = check_problem(p);
  if (s != GMM_OK) return s;
  if (p->K > p->N) return GMM_ERR_INVALID_ARG;  // K distinct rows are needed
  std::vector<int64_t> rows;
  sample_rows(p->N, p->K, seed, &rows);
  // pageable source: the copy inside gmm_init_rows has read it when that call returns
  return gmm_init_rows(p, X, rows.data(), init_var, w, mu, var, ws, ws_bytes, stream);
}

gmm_status gmm_em_step(const gmm_problem* p, const void* X, float* w, float* mu, float* var,
                       double* loglik, void* ws, size_t ws_bytes, void* stream) {
  gmm_status s = check_problem(p);
  if (s != GMM_OK) return s;
  if ((s = check_x(p, X)) != GMM_OK) return s;
  if (!w || !mu || !var) return GMM_ERR_INVALID_ARG;
  Plan P;
  if ((s = get_plan(p, ws, ws_bytes, &P)) != GMM_OK) return s;
  return em_step_impl(p, X, w, mu, var, loglik, ws, P, (cudaStream_t)stream);
}

gmm_status gmm_estep_stats(const gmm_problem* p, const void* X, const float* w, const float* mu,
                           const float* var, double* stats, void* ws, size_t ws_bytes,
                           void* stream) {
  gmm_status s = check_problem(p);
  if (s != GMM_OK) return s;
  if ((s = check_x(p, X)) != GMM_OK) return s;
  if (!w || !mu || !var || !stats) return GMM_ERR_INVALID_ARG;
  Plan P;
  if ((s = get_plan(p, ws, ws_bytes, &P)) != GMM_OK) return s;
  return estep_stats_impl(p, X, w, mu, var, stats, ws, P, (cudaStream_t)stream, p->N);
}

gmm_status gmm_mstep(const gmm_problem* p, const double* stats, int32_t nshards, float* w,
                     float* mu, float* var, double* loglik, void* stream) {
  gmm_status s = check_problem(p);
  if (s != GMM_OK) return s;
  if (!stats || !w || !mu || !var || nshards < 1) return GMM_ERR_INVALID_ARG;
  return mstep_impl(p, stats, nshards, w, mu, var, loglik, (cudaStream_t)stream);
}

gmm_status gmm_em_step_noalloc(const gmm_problem* p, const void* X, float* w, float* mu,
                               float* var, double* loglik, uint32_t* dev_flags, void* stream) {
  gmm_status s = check_problem(p);
  if (s != GMM_OK) return s;
  if ((s = check_x(p, X)) != GMM_OK) return s;
  if (!w || !mu || !var) return GMM_ERR_INVALID_ARG;
  int sms = 0;
  if ((s = device_sms(&sms)) != GMM_OK) return s;
  const Plan P = make_plan(p, sms, kNoallocScratchBytes);
  if (!P.use_tc || P.aux > kNoallocScratchBytes) {  // (the step uses no region past stats)
    fprintf(stderr,
            "gmm_em_step_noalloc: K=%d, D=%d has no tensor-core plan whose one statistics "
            "slot fits the built-in scratch of %zu bytes\n",
            p->K, p->D, kNoallocScratchBytes);
    return GMM_ERR_UNSUPPORTED;
  }
  void* ws = nullptr;
  if ((s = noalloc_scratch(&ws)) != GMM_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  unsigned int* status = (unsigned int*)ws;
  // the scratch keeps the previous call's bytes: only the status word must start at zero
  // (prep rewrites every parameter table and the fused kernel zeroes its own slot)
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), st) != cudaSuccess) {
    launch_status();
    return GMM_ERR_CUDA;
  }
  if ((s = em_step_impl(p, X, w, mu, var, loglik, ws, P, st)) != GMM_OK) return s;
  if (dev_flags && cudaMemcpyAsync(dev_flags, status, sizeof(uint32_t),
                                   cudaMemcpyDeviceToDevice, st) != cudaSuccess) {
    launch_status();
    return GMM_ERR_CUDA;
  }
  return GMM_OK;
}

gmm_status gmm_em_step_hard(const gmm_problem* p, const void* X, float* w, float* mu,
                            float* var, int32_t* labels, double* loglik, void* ws,
                            size_t ws_bytes, void* stream) {
  gmm_status s = check_problem(p);
  if (s != GMM_OK) return s;
  if ((s = check_x(p, X)) != GMM_OK) return s;
  if (!w || !mu || !var) return GMM_ERR_INVALID_ARG;
  Plan P;
  if ((s = get_plan(p, ws, ws_bytes, &P)) != GMM_OK) return s;
  if (!P.use_tc) return GMM_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  double* stats = (double*)((char*)ws + P.stats);
  if ((s = estep_stats_impl(p, X, w, mu, var, stats, ws, P, st, p->N, true, labels)) != GMM_OK)
    return s;
  return mstep_impl(p, stats, 1, w, mu, var, loglik, st);
}

gmm_status gmm_em_step_spherical(const gmm_problem* p, const void* X, float* w, float* mu,
                                 float* s2, double* loglik, void* ws, size_t ws_bytes,
                                 void* stream) {
  gmm_status s = check_problem(p);
  if (s != GMM_OK) return s;
  if ((s = check_x(p, X)) != GMM_OK) return s;
  if (!w || !mu || !s2) return GMM_ERR_INVALID_ARG;
  Plan P;
  if ((s = get_plan(p, ws, ws_bytes, &P)) != GMM_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t KD = (size_t)p->K * p->D;
  float* var = (float*)((char*)ws + P.aux);
  double* stats = (double*)((char*)ws + P.stats);
  sph_expand_kernel<<<(unsigned)((KD + 255) / 256), 256, 0, st>>>(p->D, p->K, s2, var);
  if ((s = launched(1)) != GMM_OK) return s;
  if ((s = estep_stats_impl(p, X, w, mu, var, stats, ws, P, st, p->N)) != GMM_OK) return s;
  sph_mstep_kernel<<<p->K, 128, 0, st>>>(p->N, p->D, p->K, p->var_floor, stats, w, mu, s2, loglik);
  return launched(1);
}

gmm_status gmm_kmeans_step(const gmm_problem* p, const void* X, float* centers, int32_t* labels,
                           double* inertia, void* ws, size_t ws_bytes, void* stream) {
  gmm_status s = check_problem(p);
  if (s != GMM_OK) return s;
  if ((s = check_x(p, X)) != GMM_OK) return s;
  if (!centers) return GMM_ERR_INVALID_ARG;
  Plan P;
  if ((s = get_plan(p, ws, ws_bytes, &P)) != GMM_OK) return s;
  if (!P.use_tc) return GMM_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t KD = (size_t)p->K * p->D;
  float* var = (float*)((char*)ws + P.aux);
  float* w = var + KD;
  float* v = w + p->K;
  double* stats = (double*)((char*)ws + P.stats);
  km_prep_kernel<<<1, 256, 0, st>>>(p->D, p->K, centers, w, var, v);
  if ((s = launched(1)) != GMM_OK) return s;
  if ((s = estep_stats_impl(p, X, w, centers, var, stats, ws, P, st, p->N, true, labels)) !=
      GMM_OK)
    return s;
  km_mstep_kernel<<<(unsigned)((KD + 255) / 256), 256, 0, st>>>(p->N, p->D, p->K, stats, v,
                                                                centers, inertia);
  return launched(1);
}

gmm_status gmm_fit(const gmm_problem* p, const void* X, int32_t iters, float* w, float* mu,
                   float* var, double* ll_history, void* ws, size_t ws_bytes, void* stream) {
  gmm_status s = check_problem(p);
  if (s != GMM_OK) return s;
  if ((s = check_x(p, X)) != GMM_OK) return s;
  if (!w || !mu || !var || iters < 0) return GMM_ERR_INVALID_ARG;
  Plan P;
  if ((s = get_plan(p, ws, ws_bytes, &P)) != GMM_OK) return s;
  if (iters > 0 && sf_cluster(p->N, p->D, p->K) > 0) {
    s = small_fit(p, X, iters, w, mu, var, ll_history, (unsigned int*)ws, (cudaStream_t)stream);
    if (s != GMM_ERR_UNSUPPORTED) return s;  // else: no such cluster fits now; step by step
  }
  for (int t = 0; t < iters; t++) {
    s = em_step_impl(p, X, w, mu, var, ll_history ? ll_history + t : nullptr, ws, P,
                     (cudaStream_t)stream);
    if (s != GMM_OK) return s;
  }
  return GMM_OK;
}

gmm_status gmm_loglik(const gmm_problem* p, const void* X, const float* w, const float* mu,
                      const float* var, double* loglik, void* ws, size_t ws_bytes, void* stream) {
  gmm_status s = check_problem(p);
  if (s != GMM_OK) return s;
  if ((s = check_x(p, X)) != GMM_OK) return s;
  if (!w || !mu || !var || !loglik) return GMM_ERR_INVALID_ARG;
  Plan P;
  if ((s = get_plan(p, ws, ws_bytes, &P)) != GMM_OK) return s;
  if (!P.use_tc) return GMM_ERR_UNSUPPORTED;  // no tensor-core plan for this shape
  cudaStream_t st = (cudaStream_t)stream;
  {
    char* wsb = (char*)ws;
    const TcLayout& T = P.tc;
    if ((s = tc_prep(p, w, mu, var, wsb, T, st)) != GMM_OK) return s;
    int nslots = 0;
    if ((s = tc_pass<kTcLoglik>(p, X, wsb, T, st, &nslots, loglik)) != GMM_OK) return s;
    if (T.G > 1) return GMM_OK;  // the chunks' sums went straight into *loglik
    tc_reduce_loglik_kernel<<<1, 1, 0, st>>>(p->D, p->K, (const double*)(wsb + T.slots),
                                             T.slot_stride, nslots, loglik);
    return launched(1);
  }
}

gmm_status gmm_assign_topm(const gmm_problem* p, const void* X, const float* w, const float* mu,
                           const float* var, int32_t m, int32_t* idx, float* resp, void* ws,
                           size_t ws_bytes, void* stream) {
  gmm_status s = check_problem(p);
  if (s != GMM_OK) return s;
  if ((s = check_x(p, X)) != GMM_OK) return s;
  if (!w || !mu || !var || !idx || !resp) return GMM_ERR_INVALID_ARG;
  if (m < 1 || m > kMaxTopM || m > p->K) return GMM_ERR_INVALID_ARG;
  Plan P;
  if ((s = get_plan(p, ws, ws_bytes, &P)) != GMM_OK) return s;
  if (!P.use_tc) return GMM_ERR_UNSUPPORTED;  // no tensor-core plan for this shape
  cudaStream_t st = (cudaStream_t)stream;
  if (p->xdtype == GMM_BF16)
    return tc_topm_t<__nv_bfloat16>(p, X, w, mu, var, m, idx, resp, (char*)ws, P, st);
  return tc_topm_t<float>(p, X, w, mu, var, m, idx, resp, (char*)ws, P, st);
}

gmm_status gmm_ivf_workspace_size(int64_t N, int32_t K, size_t* bytes) {
  if (!bytes || N < 1 || K < 1) return GMM_ERR_INVALID_ARG;
  if (K > kMaxK || (size_t)N > ((size_t)1 << 40)) return GMM_ERR_UNSUPPORTED;
  *bytes = ivf_layout(N, K).total;
  return GMM_OK;
}

gmm_status gmm_ivf_build(int64_t N, int32_t K, int32_t m, const int32_t* idx, const float* resp,
                         float tau, int64_t* offsets, int64_t* ids, int64_t ids_capacity,
                         void* ws, size_t ws_bytes, void* stream) {
  size_t need = 0;
  gmm_status s = gmm_ivf_workspace_size(N, K, &need);
  if (s != GMM_OK) return s;
  if (m < 1 || m > kMaxTopM || m > K) return GMM_ERR_INVALID_ARG;
  if (!idx || !resp || !offsets || !ids || isnan(tau)) return GMM_ERR_INVALID_ARG;
  if (ids_capacity < N * m) return GMM_ERR_INVALID_ARG;
  if (!ws || ((uintptr_t)ws) % 256 != 0 || ws_bytes < need) return GMM_ERR_WORKSPACE;
  const IvfLayout L = ivf_layout(N, K);
  char* b = (char*)ws;
  unsigned int* status = (unsigned int*)(b + L.status);
  int64_t* tot = (int64_t*)(b + L.tot);
  int64_t* cnt = (int64_t*)(b + L.cnt);
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemsetAsync(cnt, 0, (size_t)L.B * K * 8, st) != cudaSuccess)
    return launch_status(), GMM_ERR_CUDA;
  ivf_walk(m, false, N, K, idx, resp, tau, L, cnt, offsets, ids, status, st);
  ivf_scan_chunks_kernel<<<(K + kIvfWarps - 1) / kIvfWarps, kIvfWarps * 32, 0, st>>>(K, L.B, cnt,
                                                                                    tot);
  ivf_offsets_kernel<<<1, kIvfScanThreads, 0, st>>>(K, tot, offsets);
  ivf_walk(m, true, N, K, idx, resp, tau, L, cnt, offsets, ids, status, st);
  return launched(4);
}

gmm_status gmm_host_staging_size(const gmm_problem* p, int64_t chunk_rows, size_t* bytes) {
  gmm_status s = check_problem(p);
  if (s != GMM_OK) return s;
  if (!bytes || chunk_rows < 1) return GMM_ERR_INVALID_ARG;
  if ((size_t)chunk_rows > ((size_t)1 << 40)) return GMM_ERR_UNSUPPORTED;
  *bytes = host_staging(p, chunk_rows).total;
  return GMM_OK;
}

gmm_status gmm_em_step_host(const gmm_problem* p, const void* X_host, int64_t chunk_rows,
                            void* staging, size_t staging_bytes, float* w, float* mu, float* var,
                            double* loglik, void* ws, size_t ws_bytes, void* stream,
                            void* copy_stream) {
  size_t need = 0;
  gmm_status s = gmm_host_staging_size(p, chunk_rows, &need);
  if (s != GMM_OK) return s;
  if (!X_host || !w || !mu || !var) return GMM_ERR_INVALID_ARG;
  if (!staging || ((uintptr_t)staging) % 256 != 0 || staging_bytes < need)
    return GMM_ERR_WORKSPACE;
  if ((s = check_x(p, staging)) != GMM_OK) return s;
  Plan P;
  if ((s = get_plan(p, ws, ws_bytes, &P)) != GMM_OK) return s;
  const HostStaging H = host_staging(p, chunk_rows);
  const size_t row_bytes = (size_t)p->D * elem_bytes(p->xdtype);
  char* base = (char*)staging;
  char* buf[2] = {base, base + H.buf_bytes};
  double* total = (double*)(base + 2 * H.buf_bytes);
  double* part = (double*)(base + 2 * H.buf_bytes + H.stats_bytes);
  const size_t S = stats_doubles(p);
  cudaStream_t st = (cudaStream_t)stream, cs = (cudaStream_t)copy_stream;
  StagingEvents ev;
  if (!ev.create()) return launch_status(), GMM_ERR_CUDA;
  const char* xh = (const char*)X_host;
  const int64_t nchunks = (p->N + chunk_rows - 1) / chunk_rows;
  for (int64_t i = 0; i < nchunks; ++i) {
    const int b = (int)(i & 1);
    const int64_t r0 = i * chunk_rows;
    gmm_problem pc = *p;
    pc.N = std::min(chunk_rows, p->N - r0);
    // the copy into buffer b waits until the E-step of chunk i - 2 has read it
    if (i >= 2 && cudaStreamWaitEvent(cs, ev.used[b], 0) != cudaSuccess)
      return launch_status(), GMM_ERR_CUDA;
    if (cudaMemcpyAsync(buf[b], xh + (size_t)r0 * row_bytes, (size_t)pc.N * row_bytes,
                        cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaEventRecord(ev.copied[b], cs) != cudaSuccess ||
        cudaStreamWaitEvent(st, ev.copied[b], 0) != cudaSuccess)
      return launch_status(), GMM_ERR_CUDA;
    if ((s = estep_stats_impl(&pc, buf[b], w, mu, var, i == 0 ? total : part, ws, P, st,
                              p->N)) != GMM_OK)
      return s;
    if (i > 0) {
      stats_add_kernel<<<(unsigned)((S + 255) / 256), 256, 0, st>>>(total, part, S);
      if ((s = launched(1)) != GMM_OK) return s;
    }
    if (cudaEventRecord(ev.used[b], st) != cudaSuccess) return launch_status(), GMM_ERR_CUDA;
  }
  return mstep_impl(p, total, 1, w, mu, var, loglik, st);
}

gmm_status gmm_set_wait_budget(uint64_t ns) {
  g_wait_budget_ns = ns == 0 ? kWaitBudgetNs : ns;
  return GMM_OK;
}

gmm_status gmm_launch_count(uint64_t* count) {
  if (!count) return GMM_ERR_INVALID_ARG;
  *count = g_launches.load();
  return GMM_OK;
}

gmm_status gmm_trace_fused(void* start_event, void* stop_event) {
  if ((start_event == nullptr) != (stop_event == nullptr)) return GMM_ERR_INVALID_ARG;
  g_trace_start = (cudaEvent_t)start_event;
  g_trace_stop = (cudaEvent_t)stop_event;
  return GMM_OK;
}

gmm_status gmm_device_status(void* ws, size_t ws_bytes, void* stream, uint32_t* flags,
                             int32_t clear) {
  if (!ws || ws_bytes < 16) return GMM_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  uint32_t f = 0;
  if (cudaStreamSynchronize(st) != cudaSuccess) return launch_status(), GMM_ERR_CUDA;
  if (cudaMemcpy(&f, ws, sizeof(f), cudaMemcpyDeviceToHost) != cudaSuccess)
    return launch_status(), GMM_ERR_CUDA;
  if (clear && cudaMemset(ws, 0, sizeof(uint32_t)) != cudaSuccess)
    return launch_status(), GMM_ERR_CUDA;
  if (flags) *flags = f;
  if (f & GMM_DEVFLAG_WAIT_TIMEOUT) return GMM_ERR_TIMEOUT;
  if (f & (GMM_DEVFLAG_NONFINITE_X | GMM_DEVFLAG_BAD_PARAMS | GMM_DEVFLAG_X_RANGE))
    return GMM_ERR_NUMERIC;
  if (f & GMM_DEVFLAG_BAD_INDEX) return GMM_ERR_INVALID_ARG;
  return GMM_OK;
}

}  // extern "C"

#ifdef SCEM_PHASE_TRACE
// Performance-work builds only: copy the phase timestamps of the last
// tensor-core pass to the host.
extern "C" int scem_phase_trace_read(unsigned long long* host, int n) {
  if (n > 64 * 16) n = 64 * 16;
  return cudaMemcpyFromSymbol(host, scem::g_phase_trace, sizeof(unsigned long long) * n) ==
                 cudaSuccess
             ? 0
             : 1;
}
#endif
