// tc_em.cuh -- the fused EM pass on the 5th-generation tensor cores (sm_100a).
//
// Method: "Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering"
// (review page, section 3): per data tile, the E-step log-densities, the
// per-point log-sum-exp into responsibilities and the tile's share of the
// M-step statistics are formed on chip; only O(K*D) statistics reach memory.
//
// Expanded E-step.  With a centring vector m (the mixture mean) and a
// power-of-two scale s_d (about twice the mixture's standard deviation, so the
// scaling is exact), x^ = (x - m)/s, mu^ = (mu - m)/s, var^ = var/s^2, every
// log-joint is one dense contraction over the 2D features F = [x^, x^^2]:
//   l_nk = c_k + sum_d x^_nd a_kd + sum_d x^_nd^2 b_kd,
//   a_kd = mu^_kd / var^_kd,  b_kd = -1 / (2 var^_kd),
//   c_k  = log pi_k - 1/2 sum_d (log(2 pi var_kd) + mu^_kd^2 / var^_kd).
// F and W = [a, b] are split into fp16 pairs (hi + lo, 22 significant bits;
// each W row carries its own power-of-two scale so it sits in fp16 range) and
// the contraction takes F_hi W_hi + F_lo W_hi + F_hi W_lo (the lo*lo term is
// below fp32 rounding), accumulated in fp32 in tensor memory, starting from
// -5/8 sum_d mu^^2/var^ rather than zero (kTcStartFrac); c_k absorbs the split's
// systematic error on the component's own points (tc_prep_w_kernel).
//
// Split dimensions.  The expanded form cancels: its fp32 error grows with
// kappa_k = sum_d (mu^_kd^2 + 1) / var^_kd.  A component with kappa_k > 1e7 (in
// practice one collapsed onto a few points at the variance floor in some
// dimensions), or with kappa_k > 2e4 while it expects fewer than 50 points,
// has its dimensions with the largest shares of kappa_k -- just enough that
// the rest sum below the threshold -- taken out of the contraction (zero W).
// For each row the CUDA cores add -1/2 sum (x - mu)^2 / var over those
// dimensions, in data units from X itself (the fp16 split of x^ is too coarse
// next to a narrow dimension), onto the tensor-core log-joint of the rest,
// after a cheap filter on the tile's own features drops the rows that are
// certainly far below the best component.  Their moments, sum r (x - mu) and
// sum r (x - mu)^2 about the input means, are summed the same way (fp64
// reductions from the few rows near the component) and replace the
// tensor-core statistics of those dimensions.
//
// Statistics.  r is scaled by 2^15 and split into an fp16 pair r^ = r_hi +
// r_lo (about 22 significant bits; fp16 alone leaves components that hold a
// point or two with weight errors near 1e-3); the same r^ gives
//   N_k = sum_n r^_nk,  S1_kd = sum_n r^_nk x^_nd,  S2_kd = sum_n r^_nk x^_nd^2
// as r_hi^T (F_hi + F_lo) + r_lo^T F_hi and r^T 1 on the tensor cores,
// accumulated in fp32 in tensor memory over a few tiles and then added into
// fp64 per-cluster slots.  The variance S2/N - (S1/N)^2 magnifies the
// relative rounding error of dimension d's fp32 sums by mu^_kd^2 / var^_kd, and
// a weight is sensitive to it when the component holds few points; so the
// "precise" features (both of a dimension with mu^^2/var^ > 64, every feature
// of a component expecting fewer than 50 points) and N_k are drained after
// every tile in which the component has mass, everything every kTcDrainTiles
// tiles.  Each compute thread drains its own component (tensor-memory lane)
// with fire-and-forget fp64 reductions and zeroes what it drained in place
// with tcgen05.st, while the next tile's E-step MMAs run.  The M-step undoes
// the scales exactly.  r^ passes through one 32 KB buffer in two 64-row
// halves: rows 0-63 first, then rows 64-127 once the MMAs of the first half
// have released it.
//
// Work split.  A cluster of C = ceil(K/128) CTAs takes one 128-row tile at a
// time; CTA `rank` owns components [128 rank, 128 rank + 128).  Per tile each
// CTA converts X into F (shared memory), runs the E-step MMAs for its 128
// components (W streamed by TMA through a 3-stage ring), reduces each row's
// max / sum-exp over its components, exchanges those with the other CTAs of
// the cluster through distributed shared memory, forms r^ and runs the
// statistics MMAs.  Warps 0-7: conversion, epilogue, drains (warp w reads
// tensor-memory lanes 32(w%4)..32(w%4)+31 and component columns 64(w/4)..+63);
// warp 8: MMA issue; warp 9: TMA issue.
//
// Tensor memory (512 columns): L logits [0,128); S statistics
// [128, 128 + 64*nchunks); N_k [128 + 64*nchunks, +16).
#pragma once

#include <math.h>

#include <limits.h>

#include <algorithm>

#include "common.cuh"
#include "sm100_prims.cuh"

namespace scem {

constexpr int kTcRows = 128;      // rows per tile (= tensor-memory lanes)
constexpr int kTcComps = 128;     // components per CTA
constexpr int kTcChunk = 64;      // features per operand chunk (one swizzled 128-byte row)
constexpr int kTcStages = 3;      // depth of the W ring
constexpr int kTcMaxChunks = 4;   // features resident in shared memory: 2D <= 256
constexpr int kTcMaxD = 128;      // the largest D with resident features
// Beyond D = 128 the features stream through shared memory: kTcRoundChunks
// feature chunks (hi and lo) at a time, for the E-step and again for the
// statistics, which accumulate kTcGroupChunks chunks per pass in tensor memory
// (128 logit + 320 statistic + 16 N_k columns), one pass per feature group.
constexpr int kTcMaxDStream = 1024;
constexpr int kTcRoundChunks = 2;
constexpr uint32_t kTcRBytes = 65536;  // r^ hi | lo of a 128-row tile, streamed layout
constexpr int kTcGroupChunks = 5;
constexpr int kTcMaxCluster = 16;
constexpr int kTcThreads = 320;          // 8 compute warps + MMA warp + TMA warp
constexpr int kTcComputeThreads = 256;
constexpr int kTcMmaWarp = 8, kTcTmaWarp = 9;
constexpr int kTcDrainTiles = 8;  // tiles accumulated in fp32 before an fp64 drain
constexpr double kTcRhoPrecise = 64.0;  // mu^^2/var^ of a dimension above which its features
                                        // drain after every tile with mass
constexpr uint32_t kTcChunkBytes = 128u * 128u;  // one [128 x 64] 16-bit operand chunk
constexpr float kTcRScale = 32768.0f;            // r is stored as fp16(r * 2^15)
// Exact log-joints above this kappa_k: below it the expanded form's logit
// bias, about 4e-8 kappa_k nats with the accumulator start value below (for
// D <= 128; it grows as D / 128 beyond, and so the thresholds shrink as
// 128 / D), stays near 1e-3 nats: under the 4e-3 nats the weight tolerance
// allows, and small enough that a component's variance, which a wrong
// responsibility for a distant row shifts by that row's squared distance,
// stays within its 1e-3 tolerance ...
constexpr double kTcSharpKappa = 3e4;
constexpr double kTcSmallKappa = 6.0e3;          // ... or above this one for a component
constexpr double kTcSmallPoints = 50.0;          //     expecting fewer points than this
// Dimensions whose kappa_kd = (mu^^2 + 1)/var^ exceeds this take their moments
// in direct form (exact, fixed point) even when the contraction keeps them for
// the logits.  The tensor-core statistics give var to a relative error of
// about 1e-7 (mu^^2/var^) of the NEW variance (fp32 accumulation that rounds
// toward zero, 22-bit features); on data clipped to a range, a dimension's
// variance can shrink several-fold in one step, so the margin is wide: at 500
// the error stays near 3e-4 even after a tenfold shrink.
constexpr double kTcDirectKappa = 500.0;
// Rows whose responsibility for a component is below this add nothing to its
// direct-form moments: r (x - mu)^2 / var stays below ~2e-10 for such a row
// (its log-joint carries -(x - mu)^2 / (2 var)), negligible next to the second
// moment of a component holding ten or more points.
constexpr float kTcDirRmin = 1e-12f;
constexpr float kTcXMax = 240.0f;                // |x^| beyond this cannot be split into fp16
// Start value of the E-step accumulator, as a multiple of Q_k = sum_d mu^^2/var^.
// For a point the component explains, the linear K-steps add about +Q_k and
// the quadratic ones about -Q_k/2 (over as many accumulations), so from
// -5/8 Q_k the partial sums run -5/8 -> +3/8 -> -1/8 (in Q_k): they stay below
// Q_k in size and spend as long above zero as below it.  The tensor core's
// fp32 accumulation rounds toward zero (measured on sm_100a: its N_k errors
// follow that model, not round-to-nearest), so its errors then cancel instead
// of adding up; from zero they would grow with Q_k, which reaches 10^4 for
// tight components far from the centring point.
constexpr double kTcStartFrac = -0.625;
// Fixed-point unit of the split dimensions' direct-form moments: each row's
// r (x - mu) / sigma and r (x - mu)^2 / sigma^2 is rounded to a multiple of
// 2^-32; a warp's sum of those integers is added as a high word (q >> 32,
// signed) and a low word (q mod 2^32), each summed with a 64-bit integer
// atomic.  Integer sums do not depend on the order of the additions, so the
// result is deterministic whatever the scheduling; the rounding is 2^-33 of a
// standard deviation per row, and the low-word sum stays exact for up to 2^31
// contributing warps per component.
constexpr double kTcDirScale = 4294967296.0;  // 2^32

// kTcStats: E-step, responsibilities and statistics (with G > 1 component
//   groups, the rows' log-sum-exp comes from the groups' partials written by a
//   kTcPartial pass over the same rows).
// kTcLoglik: E-step and the log-likelihood only (one group).
// kTcPartial: E-step of this cluster's component group; each row's (max,
//   sum-exp) over the group's components goes to the row buffer.
// kTcHardStats / kTcHardPartial: the same for hard (classification) EM: each
//   row goes wholly to its most probable component (ties to the lower
//   index); the exchanged partials are (max log-joint, its component index)
//   instead of (max, sum-exp), the responsibilities one-hot, and the
//   log-likelihood the classification one, sum_n max_k l_nk.
// kTcTopm: E-step and row normalisation (with G > 1 groups, from the partial
//   pass); each (CTA, column half) writes its kTcCand largest log-joints with
//   their component indices to the candidate buffer, and the row's (max,
//   sum-exp) to the row buffer, for tc_topm_refine_kernel.
enum TcMode {
  kTcStats = 0,
  kTcLoglik = 1,
  kTcPartial = 2,
  kTcHardStats = 3,
  kTcHardPartial = 4,
  kTcTopm = 5
};
constexpr int kTcCand = 8;  // candidates per (CTA, column half) and row for top-m
__host__ __device__ constexpr bool tc_mode_stats(int m) { return m == kTcStats || m == kTcHardStats; }
__host__ __device__ constexpr bool tc_mode_partial(int m) {
  return m == kTcPartial || m == kTcHardPartial;
}
__host__ __device__ constexpr bool tc_mode_hard(int m) {
  return m == kTcHardStats || m == kTcHardPartial;
}
constexpr int kTcMaxGroups = 64;
// Largest cluster of a component group when there are several (G > 1): the
// grid must hold a whole number of clusters per group, and smaller clusters
// pack more of the SMs into it (8-CTA clusters left a third of a B200 idle).
// Measured at D = 96, K = 4096 per 1e6 rows: 8-CTA clusters (4 groups) 119 ms,
// 4 (8 groups) 92 ms, 2 (16 groups) 94 ms, 1 (32 groups) 106 ms.
constexpr int kTcGroupClusterMax = 4;
constexpr int64_t kTcChunkRowsMax = 1 << 18;       // rows per pass with component groups
constexpr size_t kTcChunkFBytesMax = 256u << 20;   // cap on the chunk's feature buffer

// Optional phase timestamps for performance work (off unless the library is
// built with -DSCEM_PHASE_TRACE): slot `idx` of the first 64 tiles of cluster
// 0, rank 0, taken by compute thread 0 or the MMA thread.
#ifdef SCEM_PHASE_TRACE
__device__ unsigned long long g_phase_trace[64 * 16];
#define SCEM_TRACE(li, idx)                                                  \
  do {                                                                       \
    if (cid == 0 && rank == 0 && (li) < 64)                                  \
      g_phase_trace[(li) * 16 + (idx)] = sm100::globaltimer_ns();            \
  } while (0)
#else
#define SCEM_TRACE(li, idx) \
  do {                      \
  } while (0)
#endif

inline int tc_nchunks(int D) { return (2 * D + kTcChunk - 1) / kTcChunk; }
inline int tc_cluster(int K) { return (K + kTcComps - 1) / kTcComps; }
__host__ __device__ inline bool tc_streamed(int nchunks) { return nchunks > kTcMaxChunks; }

// Byte offsets of the kernel's shared-memory regions (from a 1024-aligned base).
// nfb F buffers of fbytes each: two when they fit (small D), so that a tile's
// features can be written while the previous tile's statistics MMAs still
// read the other buffer.
struct TcSmem {
  uint32_t F, W, R, ONES, msm, iscs, csm, cis, wscs, cxs, mgs, shl, shs, ndc, precs, xchg, bars,
      tslot, total;
  uint32_t nfb, fbytes;
  uint32_t nr;  // feature chunks an F buffer holds: all of them, or a round when streamed
};

constexpr uint32_t kTcMaxSmem = 232448;  // 227 KB per CTA

__host__ __device__ inline TcSmem tc_smem_layout_n(int D, int C, int nchunks, uint32_t nfb) {
  TcSmem L;
  uint32_t off = 0;
  const bool streamed = tc_streamed(nchunks);
  L.nfb = nfb;
  L.nr = streamed ? (uint32_t)kTcRoundChunks : (uint32_t)nchunks;
  L.fbytes = 2u * L.nr * kTcChunkBytes;
  L.F = off;
  off += nfb * L.fbytes;
  L.W = off;
  off += kTcStages * kTcChunkBytes;
  L.R = off;
  // r^ hi | lo: one 64-row half at a time, or all 128 rows when the statistics
  // run in several rounds over the features
  off += (streamed ? 4u : 2u) * kTcChunkBytes;
  L.ONES = off;
  off += 4096;
  L.msm = off;
  off += ((uint32_t)D * 4 + 15) & ~15u;
  L.iscs = off;
  off += ((uint32_t)D * 4 + 15) & ~15u;
  L.csm = off;
  off += kTcComps * 4;
  L.cis = off;
  off += kTcComps * 4;
  L.wscs = off;
  off += kTcComps * 4;
  L.cxs = off;
  off += kTcComps * 4;
  L.mgs = off;
  off += kTcComps * 4;
  L.shl = off;
  off += (kTcComps + 8) * 4;
  L.shs = off;  // per column half: the count, then the local columns with exact log-joints
  off += 2 * (kTcComps / 2 + 1) * 4;
  L.ndc = off;  // per local component its direct dimensions, then 4 words: those with any
  off += (kTcComps + 4) * 4;
  L.precs = off;
  off += kTcComps * 4;
  L.xchg = off;
  off += 2u * 2u * C * kTcRows * 8;  // [parity][rank][column half][row]
  L.bars = off;
  off += 8 * (2 * kTcStages + 20);
  L.tslot = off;
  off += 16;
  L.total = off + 1024;  // slack for aligning the dynamic base to 1024
  return L;
}

__host__ __device__ inline TcSmem tc_smem_layout(int D, int C, int nchunks) {
  if (tc_streamed(nchunks)) return tc_smem_layout_n(D, C, nchunks, 1);
  const TcSmem two = tc_smem_layout_n(D, C, nchunks, 2);
  return two.total <= kTcMaxSmem ? two : tc_smem_layout_n(D, C, nchunks, 1);
}

// Workspace layout of the tensor-core path (after the 256-byte status block).
//   m, isc, sc : D f32 centring vector, 1/s and s (powers of two)
//   c    : C*128 f32 per-component constants of the expanded form (over the
//          dimensions the contraction keeps): the part added in the epilogue
//          (-inf for padding / pi = 0)
//   ci   : C*128 f32 the part of that constant the accumulator starts from, in
//          units of the W row scale
//   wsc  : C*128 f32 power-of-two scale of each W row
//   ndir : C*128 int32 how many of the component's leading dimensions (in perm
//          order) take their moments in direct form
//   nsplit: C*128 int32, > 0 for a component with exact log-joints
//   pmask: [C*128 x Fpad/32] u32 per feature of each component, 1 if it is
//          drained after every tile with mass (see tc_prep_w_kernel)
//   perm : [C*128 x D] u16 dimensions of each component by decreasing
//          (mu^^2 + 1)/var^
//   muh, ph : [C*128 x D] f32 mu and 1/var (data units) in perm order
//   mun, pn : [C*128 x D] f32 mu and 1/var (data units) in natural order
//   cx   : C*128 f32 log pi_k - 1/2 sum_d log(2 pi var_kd): the direct form's constant
//   mg   : C*128 f32 bound on the error of the contraction's log-joint of a
//          component with exact log-joints (see tc_prep_w_kernel), 0 for the others
//   whi, wlo : [C*128 x 64*nchunks] fp16 operand W (hi and lo parts)
//   rank : [C*128 x D] u16 position of each dimension in perm
//   dirq : [C*128 x 4D] u64 direct-form moments of split dimensions about the
//          input means, by perm position i, as 64-bit fixed-point words (see
//          kTcDirScale): per component, words i / D+i hold the high / low
//          words of sum r (x - mu) / sigma, words 2D+i / 3D+i those of
//          sum r (x - mu)^2 / sigma^2.  One area for all clusters: integer
//          additions commute, so the sums do not depend on the order in which
//          rows or clusters add them.  Zeroed by tc_prep_w_kernel.
//   slots: P per-cluster slots of slot_stride doubles:
//          [(2D+1) x K] feature-major statistics (S1 rows 0..D-1, S2 rows
//          D..2D-1, N_k row 2D), then the cluster's LL.
//   With G > 1 component groups, also (after the slots):
//   fhi, flo : [R x Fpad] fp16 features [x^, x^^2] (hi and lo parts) of one
//              chunk of R rows, written by tc_convert_kernel, read by TMA
//   part     : [R x G] float2 (max, sum-exp) of each row over each group
//   rbuf     : streamed features with several statistics groups: [R/128 x G C]
//              r^ images (kTcRBytes) of a chunk's tiles, written by the first
//              group's pass and read by the others
//   Top-m assignment, for chunks of Rt rows:
//   cand     : [Rt x (G C 2) x kTcCand] float2 (log-joint, index) candidates
//   rowst    : [Rt] float2 (max, sum-exp) of each row
struct TcLayout {
  size_t m, isc, sc, c, ci, wsc, cx, mg, ndir, nsplit, precise, pmask, muh, ph, perm, rank, mun, pn,
      whi,
      wlo, dirq, slots, fhi, flo, part, rbuf, cand, rowst, total, slot_stride;
  int C, G, nchunks, Kpad, Fpad, P;
  int nfg, NFG;  // feature chunks per statistics group, and groups (1 unless streamed)
  int64_t R;   // rows per chunk (G > 1, or streamed features)
  int64_t Rt;  // rows per chunk of the top-m assignment
};

// Cluster size C and number of component groups G for a shape: the fewest
// groups whose cluster (C = ceil(ceil(K/128) / G) CTAs of 128 components, at
// most 16) fits the kernel's shared memory, and no more groups than the SMs
// can hold one cluster each.  False if none does (or D is not a multiple of 4
// up to 128): such shapes run on the CUDA cores.
inline bool tc_shape(int D, int K, int num_sms, int* C_out, int* G_out) {
  if (!(D >= 4 && D <= kTcMaxDStream && D % 4 == 0 && K >= 1)) return false;
  const int cfull = tc_cluster(K);
  for (int G = 1; G <= kTcMaxGroups; G++) {
    const int C = (cfull + G - 1) / G;
    if (C > kTcMaxCluster || (G > 1 && C > kTcGroupClusterMax)) continue;
    if (tc_smem_layout(D, C, tc_nchunks(D)).total > kTcMaxSmem) continue;
    if (G > 1 && num_sms / C < G) return false;
    *C_out = C;
    *G_out = G;
    return true;
  }
  return false;
}

inline bool tc_shape_ok(int D, int K, int num_sms = 148) {
  int C, G;
  return tc_shape(D, K, num_sms, &C, &G);
}

// Rows per chunk with component groups: at most 2^18, the chunk's features
// (4 Fpad bytes per row) at most 256 MiB, a multiple of the tile.
inline int64_t tc_chunk_rows(int Fpad) {
  int64_t r = (int64_t)(kTcChunkFBytesMax / (4u * (size_t)Fpad));
  r = std::min<int64_t>(r, kTcChunkRowsMax);
  return r / kTcRows * kTcRows;
}

inline TcLayout tc_layout(int D, int K, int num_sms, size_t cap = 0) {
  TcLayout L;
  L.C = 1;
  L.G = 1;
  tc_shape(D, K, num_sms, &L.C, &L.G);
  L.nchunks = tc_nchunks(D);
  L.Kpad = L.G * L.C * kTcComps;
  L.Fpad = L.nchunks * kTcChunk;
  const bool streamed = tc_streamed(L.nchunks);
  L.nfg = streamed ? kTcGroupChunks : L.nchunks;
  L.NFG = (L.nchunks + L.nfg - 1) / L.nfg;
  L.R = (L.G > 1 || streamed) ? tc_chunk_rows(L.Fpad) : 0;
  if (streamed && L.NFG > 1) {  // the r^ images of a chunk (4 Kpad bytes a row) at most 256 MiB
    const int64_t rr = (int64_t)(kTcChunkFBytesMax / (4u * (size_t)L.Kpad)) / kTcRows * kTcRows;
    L.R = std::max<int64_t>(kTcRows, std::min<int64_t>(L.R, rr));
  }
  size_t off = 256;
  L.m = off;
  off = align_up(off + (size_t)D * 4, 256);
  L.isc = off;
  off = align_up(off + (size_t)D * 4, 256);
  L.sc = off;
  off = align_up(off + (size_t)D * 4, 256);
  L.c = off;
  off = align_up(off + (size_t)L.Kpad * 4, 256);
  L.ci = off;
  off = align_up(off + (size_t)L.Kpad * 4, 256);
  L.wsc = off;
  off = align_up(off + (size_t)L.Kpad * 4, 256);
  L.cx = off;
  off = align_up(off + (size_t)L.Kpad * 4, 256);
  L.mg = off;
  off = align_up(off + (size_t)L.Kpad * 4, 256);
  L.ndir = off;
  off = align_up(off + (size_t)L.Kpad * 4, 256);
  L.nsplit = off;
  off = align_up(off + (size_t)L.Kpad * 4, 256);
  L.muh = off;
  off = align_up(off + (size_t)L.Kpad * D * 4, 256);
  L.ph = off;
  off = align_up(off + (size_t)L.Kpad * D * 4, 256);
  L.perm = off;
  off = align_up(off + (size_t)L.Kpad * D * 2, 256);
  L.rank = off;
  off = align_up(off + (size_t)L.Kpad * D * 2, 256);
  L.mun = off;
  off = align_up(off + (size_t)L.Kpad * D * 4, 256);
  L.pn = off;
  off = align_up(off + (size_t)L.Kpad * D * 4, 256);
  L.whi = off;
  off = align_up(off + (size_t)L.Kpad * L.Fpad * 2, 256);
  L.wlo = off;
  off = align_up(off + (size_t)L.Kpad * L.Fpad * 2, 256);
  L.precise = off;
  off = align_up(off + (size_t)L.Kpad * 4, 256);
  L.pmask = off;
  off = align_up(off + (size_t)L.Kpad * (L.Fpad / 32) * 4, 256);
  L.dirq = off;
  off = align_up(off + (size_t)4 * D * L.Kpad * 8, 256);
  L.slot_stride = align_up((size_t)(2 * D + 1) * K + 1, 32);
  // the chunk buffers of pre-converted features (G > 1 or streamed), ahead of the slots
  L.fhi = L.flo = L.part = off;
  if (L.R > 0) {
    L.fhi = off;
    off = align_up(off + (size_t)L.R * L.Fpad * 2, 256);
    L.flo = off;
    off = align_up(off + (size_t)L.R * L.Fpad * 2, 256);
    L.part = off;
    off = align_up(off + (size_t)L.R * L.G * 8, 256);
  }
  // streamed features with several statistics groups: the r^ image of every
  // (tile, CTA) of a chunk, stored by the first group's pass
  L.rbuf = off;
  if (streamed && L.NFG > 1)
    off = align_up(off + (size_t)(L.R / kTcRows) * (L.Kpad / kTcComps) * kTcRBytes, 256);
  // top-m candidates: at most 64 MiB, at most 2^18 rows (and R with groups);
  // one tile's worth under a byte cap (the no-allocation step runs no top-m)
  {
    const size_t per_row = (size_t)L.G * L.C * 2 * kTcCand * 8 + 8;
    int64_t rt = (int64_t)((size_t)(64u << 20) / per_row) / kTcRows * kTcRows;
    rt = std::max<int64_t>(kTcRows, std::min<int64_t>(rt, kTcChunkRowsMax));
    if (L.R > 0) rt = std::min<int64_t>(rt, L.R);
    if (cap) rt = kTcRows;
    L.Rt = rt;
    L.cand = off;
    off = align_up(off + (size_t)rt * (per_row - 8), 256);
    L.rowst = off;
    off = align_up(off + (size_t)rt * 8, 256);
  }
  L.slots = off;
  // one slot per cluster; with G > 1 a whole number of clusters per group
  L.P = num_sms / L.C;
  if (cap) {
    const size_t per = L.slot_stride * 8;
    const size_t fit = cap > off ? (cap - off) / per : 0;
    if ((size_t)L.P > fit) L.P = (int)fit;
  }
  L.P = L.P / L.G * L.G;
  L.total = align_up(off + (size_t)L.P * L.slot_stride * 8, 256);
  return L;
}

struct TcArgs {
  const void* X;
  int64_t N;
  int D, K, C, nchunks;
  const float* m;       // centring vector, D
  const float* isc;     // 1/s, D
  const float* c;       // expanded-form constants added in the epilogue, C*128
                        // (-inf for padding / pi = 0)
  const float* ci;      // accumulator start values (W-row-scale units), C*128
  const float* wsc;     // W row scales, C*128
  const int* ndir;      // leading perm dimensions with direct-form moments, C*128
  const int* nsplit;    // > 0: the component takes exact log-joints, C*128
  const float* muh;     // mu (data units) in perm order, C*128 x D
  const float* ph;      // 1/var (data units) in perm order, C*128 x D
  const uint16_t* perm;  // dimensions by decreasing (mu^^2 + 1)/var^, C*128 x D
  const float* mun;     // mu (data units), C*128 x D
  const float* pn;      // 1/var (data units), C*128 x D
  const float* cx;      // direct-form constants, C*128
  const float* mg;      // error bounds of the contraction's log-joints, C*128
  double* slots;        // per-cluster statistic slots
  size_t slot_stride;   // doubles per slot: (2D+1)*K statistics + LL
  unsigned long long* dirq;  // fixed-point direct-form moments of split dimensions, 4D x Kpad
  int Kpad;
  int G;                // component groups; cluster c serves group c % G
  float2* part;         // G > 1: [rows x G] (max, sum-exp) per row and group
  int accumulate;       // 1: add onto the slots (a later chunk of the same step)
  int32_t* labels;      // hard EM: each row's component (may be null)
  float2* cand;         // top-m: [rows x (G C 2) x kTcCand] (log-joint, index) candidates
  float2* rowst;        // top-m: [rows] the row's (max, sum-exp) over all components
  int ncand;            // top-m: candidates kept per (CTA, column half), <= kTcCand
  int fg0, nfgc, nfg;   // streamed features: this pass's statistics group (first chunk,
                        // chunks) and the group size that lays out tensor memory
  uint8_t* rbuf;        // streamed features with several statistics groups: the r^
                        // image of every (tile, CTA) of the chunk, kTcRBytes each
  int rmode;            // 0; 1: the first group's pass stores r^ to rbuf; 2: a later
                        // group's pass loads it instead of repeating the E-step
  unsigned int* status;
  int drain_tiles;
  const int* precise;   // 1: some feature of the component is drained every tile, C*128
  const uint32_t* pmask;  // which features, C*128 x (Fpad/32) words
  uint64_t wait_ns;   // budget of every wait for another warp or CTA (gmm_set_wait_budget)
  uint64_t drain_ns;  // budget of the two waits for the CTA's own copies and MMAs in flight
                      // before it may release shared and tensor memory (fixed, 1 s): these
                      // complete in microseconds and ignore the abort bit
};

// A shared-memory descriptor advanced by `bytes` (start-address field only;
// every operand lies within the first 256 KB of shared memory, so no carry).
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float round_half(float a) { return __half2float(__float2half_rn(a)); }

// (a, b) -> fp16 pairs hi = fp16(a, b) and lo = fp16(a - hi_a, b - hi_b), packed:
// three conversion instructions for two values.
__device__ __forceinline__ void split_half2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(a, b);
  const float2 f = __half22float2(h);
  const __half2 l = __floats2half2_rn(a - f.x, b - f.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

template <typename XT>
__device__ __forceinline__ void load4(const XT* X, size_t i, float (&x)[4]);
template <>
__device__ __forceinline__ void load4<float>(const float* X, size_t i, float (&x)[4]) {
  const float4 v = __ldg(reinterpret_cast<const float4*>(X + i));
  x[0] = v.x;
  x[1] = v.y;
  x[2] = v.z;
  x[3] = v.w;
}
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* X, size_t i,
                                                      float (&x)[4]) {
  const uint2 v = __ldg(reinterpret_cast<const uint2*>(X + i));
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&v.x);
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&v.y);
  x[0] = __low2float(a);
  x[1] = __high2float(a);
  x[2] = __low2float(b);
  x[3] = __high2float(b);
}

template <typename XT>
__device__ __forceinline__ float load1(const XT* X, int i);
template <>
__device__ __forceinline__ float load1<float>(const float* X, int i) {
  return __ldg(X + i);
}
template <>
__device__ __forceinline__ float load1<__nv_bfloat16>(const __nv_bfloat16* X, int i) {
  return __bfloat162float(X[i]);
}

// 10 warps put 3 on some of the 4 sub-partitions (16K registers each): 168 registers
// per thread at most.
// FSRC = 0: the compute warps convert X into the features F in shared memory.
// FSRC = 1: F comes pre-converted (tc_convert_kernel) and the TMA warp loads
//           each tile's F chunks (tm_fhi / tm_flo) next to the W stream.
template <typename XT, int MODE, int FSRC>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_fused_kernel(const TcArgs a, const __grid_constant__ CUtensorMap tm_whi,
                    const __grid_constant__ CUtensorMap tm_wlo,
                    const __grid_constant__ CUtensorMap tm_fhi,
                    const __grid_constant__ CUtensorMap tm_flo) {
  using namespace sm100;
  constexpr bool kStats = tc_mode_stats(MODE), kPartial = tc_mode_partial(MODE);
  constexpr bool kHard = tc_mode_hard(MODE);
  // A pass without statistics on pre-converted features overlaps tiles: two
  // logit buffers in tensor memory (columns [0, 128) and [128, 256), free of
  // statistics here), so the E-step of tile i+1 runs while the epilogue of
  // tile i reads the other buffer; the F buffer is released as soon as the
  // E-step is done with it.
  constexpr bool kOverlap = !kStats && FSRC;
  // Streamed features with several statistics groups: the first group's pass
  // stores each tile's r^ image, the later groups' passes load it instead of
  // repeating the E-step and its epilogue.
  const bool rstore = kStats && FSRC == 2 && a.rmode == 1;
  const bool rload = kStats && FSRC == 2 && a.rmode == 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const int D = a.D, K = a.K, C = a.C, nch = a.nchunks;
  const TcSmem L = tc_smem_layout(D, C, nch);
  uint8_t* sF = sm + L.F;  // [hi|lo][chunk] x [128 rows x 64 features]
  uint8_t* sW = sm + L.W;  // ring of [128 components x 64 features]
  uint8_t* sR = sm + L.R;  // r_hi | r_lo, each [64 rows] x [128 components] (two 64-wide MN atoms)
  uint8_t* sOnes = sm + L.ONES;
  float* msm = reinterpret_cast<float*>(sm + L.msm);
  float* iscs = reinterpret_cast<float*>(sm + L.iscs);
  float* csm = reinterpret_cast<float*>(sm + L.csm);
  float* cis = reinterpret_cast<float*>(sm + L.cis);
  float* wscs = reinterpret_cast<float*>(sm + L.wscs);
  float* cxs = reinterpret_cast<float*>(sm + L.cxs);
  float* mgs = reinterpret_cast<float*>(sm + L.mgs);
  // [0]: how many local components take exact log-joints or direct-form
  // moments; [129..132]: bit j of word q marks local component 32q + j as one
  // with exact log-joints
  int* shl = reinterpret_cast<int*>(sm + L.shl);
  int* shs = reinterpret_cast<int*>(sm + L.shs);  // [half][0] = count, [half][1..] = columns
  int* ndc = reinterpret_cast<int*>(sm + L.ndc);  // [128] direct dimensions, [128..131] mask
  int* precs = reinterpret_cast<int*>(sm + L.precs);
  float2* xchg = reinterpret_cast<float2*>(sm + L.xchg);  // [2][C][2][128] (max, sum-exp)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* full = bars;
  uint64_t* empty = bars + kTcStages;
  uint64_t* f_full = bars + 2 * kTcStages;
  uint64_t* l_full = f_full + 1;
  uint64_t* r_full = f_full + 2;
  uint64_t* s_done = f_full + 3;
  uint64_t* drained = f_full + 4;
  uint64_t* xbar = f_full + 5;  // [2]
  uint64_t* final_bar = f_full + 7;
  uint64_t* r_full1 = f_full + 8;  // second 64-row half of r^ written
  uint64_t* r_free = f_full + 9;   // MMAs of the first half done with the r^ buffer
  uint64_t* cbar = f_full + 10;    // rendezvous of the 256 compute threads
  uint64_t* f_free = f_full + 11;  // [2] FSRC = 1: MMAs and epilogue done with an F buffer
  uint64_t* f_tx = f_full + 13;    // [2] FSRC = 1: an F buffer's TMA loads have landed
  uint64_t* f_full2 = f_full + 15;  // [2] overlap: start values in logit buffer b stored
  uint64_t* l_full2 = f_full + 17;  // [2] overlap: E-step into logit buffer b done
  uint64_t* r_tx = f_full + 19;     // rmode 2: a tile's r^ loaded from rbuf

  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L.tslot);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  // cluster c serves component group c % G and takes every (nclusters/G)-th tile
  const uint32_t ngrp = (uint32_t)a.G;
  const uint32_t grp = cluster_id_x() % ngrp;
  const uint32_t cid = cluster_id_x() / ngrp, ncl = nclusters_x() / ngrp;
  const uint32_t slot_id = cluster_id_x();
  const int64_t ntiles = (a.N + kTcRows - 1) / kTcRows;
  const int64_t my_tiles = ((int64_t)cid < ntiles) ? (ntiles - 1 - (int64_t)cid) / ncl + 1 : 0;
  const int k0 = (int)(grp * (uint32_t)C + rank) * kTcComps;
  volatile unsigned int* status = a.status;
  constexpr unsigned int kAbort = GMM_DEVFLAG_WAIT_TIMEOUT;
  double* slot = a.slots + (size_t)slot_id * a.slot_stride;
  const size_t ll_index = (size_t)(2 * D + 1) * K;

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    for (int s = 0; s < kTcStages; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(f_full, kTcComputeThreads);  // start values stored (and, FSRC = 0, F written)
    for (int b = 0; b < 2; b++) {
      mbar_init(&f_free[b], 1);
      mbar_init(&f_tx[b], 1);
      mbar_init(&f_full2[b], kTcComputeThreads);
      mbar_init(&l_full2[b], 1);
    }
    mbar_init(r_tx, 1);

    mbar_init(l_full, 1);
    mbar_init(r_full, kTcComputeThreads / 2);
    mbar_init(r_full1, kTcComputeThreads / 2);
    mbar_init(r_free, 1);
    mbar_init(s_done, 1);
    mbar_init(drained, kTcComputeThreads);
    mbar_init(cbar, kTcComputeThreads);
    mbar_init(&xbar[0], (uint32_t)C * (kTcComputeThreads / 32));  // one arrive per warp
    mbar_init(&xbar[1], (uint32_t)C * (kTcComputeThreads / 32));
    mbar_init(final_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  for (int i = tid; i < D; i += kTcThreads) {
    msm[i] = a.m[i];
    iscs[i] = a.isc[i];
  }
  for (int i = tid; i < kTcComps; i += kTcThreads) {
    csm[i] = a.c[k0 + i];
    cis[i] = a.ci[k0 + i];
    wscs[i] = a.wsc[k0 + i];
    cxs[i] = a.cx[k0 + i];
    mgs[i] = a.mg[k0 + i];
    precs[i] = a.precise[k0 + i];
  }
  if (tid == 0) {
    int n = 0;
    uint32_t mw[4] = {0u, 0u, 0u, 0u};
    for (int j = 0; j < kTcComps; j++)
      if (a.ndir[k0 + j] > 0 || a.nsplit[k0 + j] > 0) {
        n++;
        if (a.nsplit[k0 + j] > 0) mw[j >> 5] |= 1u << (j & 31);
      }
    shl[0] = n;
    for (int q = 0; q < 4; q++) shl[kTcComps + 1 + q] = (int)mw[q];
    // per column half, the columns with exact log-joints
    for (int h = 0; h < 2; h++) {
      int c = 0;
      for (int j = 64 * h; j < 64 * h + 64; j++)
        if ((mw[j >> 5] >> (j & 31)) & 1u) shs[h * (kTcComps / 2 + 1) + 1 + c++] = j;
      shs[h * (kTcComps / 2 + 1)] = c;
    }
    // per local component its direct dimensions, and which have any
    uint32_t dw[4] = {0u, 0u, 0u, 0u};
    for (int j = 0; j < kTcComps; j++) {
      ndc[j] = a.ndir[k0 + j];
      if (ndc[j] > 0) dw[j >> 5] |= 1u << (j & 31);
    }
    for (int q = 0; q < 4; q++) ndc[kTcComps + q] = (int)dw[q];
  }
  for (int i = tid; i < 2048; i += kTcThreads)
    reinterpret_cast<__half*>(sOnes)[i] = __float2half_rn(1.0f);
  // padding features of F must read as zero in every MMA (FSRC = 1: the
  // pre-converted features hold zeros there)
  if (!FSRC)
    for (uint32_t i = tid; i < L.nfb * L.fbytes / 16; i += kTcThreads)
      reinterpret_cast<uint4*>(sF)[i] = make_uint4(0, 0, 0, 0);
  if (kStats && !a.accumulate) {
    for (int f = 0; f <= 2 * D; f++)
      for (int kk = tid; kk < kTcComps; kk += kTcThreads)
        if (k0 + kk < K) slot[(size_t)f * K + k0 + kk] = 0.0;
  }
  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync();
  tc_fence_after_sync();
  const uint32_t tmem = *tslot;
  const uint32_t tL = tmem;
  const uint32_t tS = tmem + 128;
  const uint32_t tNK = tmem + 128 + 64 * (uint32_t)(FSRC == 2 ? a.nfg : nch);

  if (warp == kTcTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_whi);
      tma_prefetch_desc(&tm_wlo);
      if (FSRC) {
        tma_prefetch_desc(&tm_fhi);
        tma_prefetch_desc(&tm_flo);
      }
      uint32_t stage = 0, phase = 0;
      int64_t issued = 0, fissued = 0, rissued = 0;
      for (int64_t li = 0; li < my_tiles; li++) {
        bool ok = true;
        // FSRC = 1: this tile's features into F buffer b, once the tile that
        // used it last (li - nfb) is done with it.  Issued after the tile's
        // first W stages, which the ring can take before that.
        auto load_features = [&]() -> bool {
          const uint32_t b = (uint32_t)(li % L.nfb);
          const int64_t use = li / L.nfb;
          if (use > 0 && !mbar_wait_bounded(&f_free[b], (uint32_t)((use - 1) & 1), status,
                                            kAbort, a.wait_ns))
            return false;
          const int y = (int)(((int64_t)cid + li * ncl) * kTcRows);
          uint8_t* dst = sF + b * L.fbytes;
          mbar_arrive_expect_tx(&f_tx[b], 2u * (uint32_t)nch * kTcChunkBytes);
          for (int c = 0; c < nch; c++) {
            tma_load_2d(dst + (uint32_t)c * kTcChunkBytes, &tm_fhi, c * kTcChunk, y, &f_tx[b]);
            tma_load_2d(dst + (uint32_t)(nch + c) * kTcChunkBytes, &tm_flo, c * kTcChunk, y,
                        &f_tx[b]);
          }
          fissued++;
          return true;
        };
        // FSRC = 2: the features stream through the one F buffer a round of
        // chunks [c0, c0 + n) at a time (u counts the buffer's uses)
        auto load_round = [&](int c0, int n) -> bool {
          if (fissued > 0 && !mbar_wait_bounded(&f_free[0], (uint32_t)((fissued - 1) & 1),
                                                status, kAbort, a.wait_ns))
            return false;
          const int y = (int)(((int64_t)cid + li * ncl) * kTcRows);
          mbar_arrive_expect_tx(&f_tx[0], 2u * (uint32_t)n * kTcChunkBytes);
          for (int c = 0; c < n; c++) {
            tma_load_2d(sF + (uint32_t)c * kTcChunkBytes, &tm_fhi, (c0 + c) * kTcChunk, y,
                        &f_tx[0]);
            tma_load_2d(sF + (L.nr + (uint32_t)c) * kTcChunkBytes, &tm_flo, (c0 + c) * kTcChunk,
                        y, &f_tx[0]);
          }
          fissued++;
          return true;
        };
        if (rload) {
          // the tile's r^ image, once the previous tile's statistics MMAs are
          // done with the buffer, then the statistics group's feature rounds
          if (li > 0 && !mbar_wait_bounded(s_done, (uint32_t)((li - 1) & 1), status, kAbort,
                                           a.wait_ns))
            break;
          const uint8_t* src =
              a.rbuf + ((size_t)(((int64_t)cid + li * ncl) * ngrp + grp) * C + rank) * kTcRBytes;
          mbar_arrive_expect_tx(r_tx, kTcRBytes);
          for (uint32_t q = 0; q < kTcRBytes; q += 16384u)
            bulk_load(sR + q, src + q, 16384u, r_tx);
          rissued++;
          for (int c = a.fg0; c < a.fg0 + a.nfgc && ok; c += (int)L.nr)
            ok = load_round(c, min((int)L.nr, a.fg0 + a.nfgc - c));
          if (!ok) break;
          continue;
        }
        int wi = 0;  // W loads issued for this tile
        for (int c = 0; c < nch && ok; c++)
          for (int part = 0; part < 2 && ok; part++, wi++) {
            if (FSRC == 2 && part == 0 && c % (int)L.nr == 0)
              ok = load_round(c, min((int)L.nr, nch - c));
            if (FSRC == 1 && wi == (2 * nch < kTcStages ? 2 * nch : kTcStages))
              ok = load_features();
            if (!ok) break;
            ok = mbar_wait_bounded(&empty[stage], phase ^ 1u, status, kAbort, a.wait_ns);
            if (!ok) break;
            mbar_arrive_expect_tx(&full[stage], kTcChunkBytes);
            tma_load_2d(sW + stage * kTcChunkBytes, part ? &tm_wlo : &tm_whi, c * kTcChunk, k0,
                        &full[stage]);
            issued++;
            if (++stage == kTcStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
        if (ok && FSRC == 1 && wi <= kTcStages && wi == 2 * nch) ok = load_features();
        // FSRC = 2: the statistics group's chunks once more, for the statistics MMAs
        if (FSRC == 2 && kStats)
          for (int c = a.fg0; c < a.fg0 + a.nfgc && ok; c += (int)L.nr)
            ok = load_round(c, min((int)L.nr, a.fg0 + a.nfgc - c));
        if (!ok) break;
      }
      // every load issued must have landed before the CTA may exit
      for (int s = 0; s < kTcStages && s < issued; s++) {
        const int64_t uses = (issued - s + kTcStages - 1) / kTcStages;  // loads into stage s
        mbar_wait_bounded(&full[s], (uint32_t)((uses - 1) & 1), status, 0u, a.drain_ns);
      }
      for (int b = 0; b < (int)L.nfb && b < fissued; b++) {
        const int64_t uses = (fissued - b + L.nfb - 1) / L.nfb;  // feature loads into buffer b
        mbar_wait_bounded(&f_tx[b], (uint32_t)((uses - 1) & 1), status, 0u, a.drain_ns);
      }
      if (rissued > 0) mbar_wait_bounded(r_tx, (uint32_t)((rissued - 1) & 1), status, 0u, a.drain_ns);
    }
  } else if (warp == kTcMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idE = idesc_f16_f32(128, 128, false, false);
      // one statistics MMA covers all 64*nch features: the chunks are MN atoms 16 KB apart
      const uint32_t idS = idesc_f16_f32(128, 64 * nch, true, true);
      const uint32_t idN = idesc_f16_f32(128, 16, true, false);
      const uint32_t fb = smem_u32(sF), wb = smem_u32(sW), rb = smem_u32(sR);
      const uint32_t ob = smem_u32(sOnes);
      const uint64_t dF = sw128_desc(fb, 16, 1024);        // F as the K-major E-step A operand
      const uint64_t dW = sw128_desc(wb, 16, 1024);        // W stage as the E-step B operand
      const uint64_t dFs = sw128_desc(fb, 16384, 1024);    // F as the MN-major statistics B
      const uint64_t dR = sw128_desc(rb, 8192, 1024);      // r^ as the MN-major statistics A
      const uint64_t dOnes = sw128_desc(ob, 16, 1024);
      uint32_t stage = 0, phase = 0, ndrain = 0;
      int64_t fu = 0;  // FSRC = 2: uses of the F buffer so far (rounds)
      // FSRC = 2: the statistics MMAs of tile li over this pass's feature
      // group, a round of chunks at a time, once the previous tile's drain is done
      auto stats_streamed = [&](int64_t li) -> bool {
        if (li > 0) {
          if (!mbar_wait_bounded(drained, ndrain & 1u, status, kAbort, a.wait_ns)) return false;
          ndrain++;
        }
        tc_fence_after_sync();
        const bool first = li == 0;
        for (int c0 = a.fg0; c0 < a.fg0 + a.nfgc; c0 += (int)L.nr) {
          const int n = min((int)L.nr, a.fg0 + a.nfgc - c0);
          if (!mbar_wait_bounded(&f_tx[0], (uint32_t)(fu & 1), status, kAbort, a.wait_ns))
            return false;
          tc_fence_after_sync();
          const uint32_t idSr = idesc_f16_f32(128, 64 * n, true, true);
          const uint32_t tSr = tS + 64u * (uint32_t)(c0 - a.fg0);
#pragma unroll 1
          for (int k8 = 0; k8 < 8; k8++) {  // 16-row K-steps over the 128 rows
            const uint32_t hofs = 32768u * (uint32_t)(k8 >> 2);
            const uint64_t ahi = desc_add(dR, hofs + 2048u * (k8 & 3));
            const uint64_t alo = desc_add(dR, hofs + 16384u + 2048u * (k8 & 3));
            const bool acc = !(first && k8 == 0);
            const uint32_t kr = 2048u * (uint32_t)k8;  // F rows of this K-step
            const uint64_t fhi = desc_add(dFs, kr);
            const uint64_t flo = desc_add(dFs, L.nr * kTcChunkBytes + kr);
            mma_bf16(tSr, ahi, fhi, idSr, acc);
            mma_bf16(tSr, ahi, flo, idSr, true);
            mma_bf16(tSr, alo, fhi, idSr, true);
            if (c0 == a.fg0) {
              mma_bf16(tNK, ahi, dOnes, idN, acc);
              mma_bf16(tNK, alo, dOnes, idN, true);
            }
          }
          mma_commit(&f_free[0]);
          fu++;
        }
        return true;
      };
      for (int64_t li = 0; li < my_tiles; li++) {
        if (rload) {
          // r^ from the first group's pass: the statistics MMAs only
          if (!mbar_wait_bounded(r_tx, (uint32_t)(li & 1), status, kAbort, a.wait_ns)) break;
          if (!stats_streamed(li)) break;
          mma_commit(s_done);
          continue;
        }
        const uint32_t lb = kOverlap ? (uint32_t)(li & 1) : 0u;  // logit buffer
        const uint32_t tLb = tL + 128u * lb;
        if (kOverlap) {
          if (!mbar_wait_bounded(&f_full2[lb], (uint32_t)((li >> 1) & 1), status, kAbort,
                                 a.wait_ns))
            break;
        } else if (!mbar_wait_bounded(f_full, (uint32_t)(li & 1), status, kAbort, a.wait_ns)) {
          break;
        }
        if (FSRC == 1 && !mbar_wait_bounded(&f_tx[li % L.nfb], (uint32_t)((li / L.nfb) & 1),
                                            status, kAbort, a.wait_ns))
          break;
        SCEM_TRACE(li, 8);
        tc_fence_after_sync();
        bool ok = true;
        const uint32_t fofs = (uint32_t)(li % L.nfb) * L.fbytes;  // this tile's F buffer
        for (int c = 0; c < nch && ok; c++) {
          // FSRC = 2: chunk c sits in slot c mod nr of the round buffer
          const uint32_t cs = FSRC == 2 ? (uint32_t)c % L.nr : (uint32_t)c;
          if (FSRC == 2 && cs == 0) {
            ok = mbar_wait_bounded(&f_tx[0], (uint32_t)(fu & 1), status, kAbort, a.wait_ns);
            if (!ok) break;
            tc_fence_after_sync();
          }
          const uint32_t fhi = fb + fofs + cs * kTcChunkBytes;
          const uint32_t flo = fb + fofs + (L.nr + cs) * kTcChunkBytes;
          for (int part = 0; part < 2; part++) {
            ok = mbar_wait_bounded(&full[stage], phase, status, kAbort, a.wait_ns);
            if (!ok) break;
            tc_fence_after_sync();
            const uint64_t wd = desc_add(dW, stage * kTcChunkBytes);
            const uint64_t fhd = desc_add(dF, fhi - fb), fld = desc_add(dF, flo - fb);
#pragma unroll
            for (int ks = 0; ks < 4; ks++) {
              const uint64_t bd = desc_add(wd, 32u * ks);
              mma_bf16(tLb, desc_add(fhd, 32u * ks), bd, idE, true);  // onto the start values
              if (part == 0) mma_bf16(tLb, desc_add(fld, 32u * ks), bd, idE, true);
            }
            mma_commit(&empty[stage]);
            if (++stage == kTcStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
          // FSRC = 2: the round's last chunk is issued; the buffer is free once it is done
          if (FSRC == 2 && ok && (cs + 1 == L.nr || c + 1 == nch)) {
            mma_commit(&f_free[0]);
            fu++;
          }
        }
        if (!ok) break;
        if (kOverlap) {
          mma_commit(&l_full2[lb]);
          // the F buffer is free once the E-step is done with it (the epilogue
          // reads X, not F)
          if (FSRC == 1) mma_commit(&f_free[li % L.nfb]);
          continue;
        }
        mma_commit(l_full);
        SCEM_TRACE(li, 9);
        if (!mbar_wait_bounded(r_full, (uint32_t)(li & 1), status, kAbort, a.wait_ns)) break;
        SCEM_TRACE(li, 10);
        tc_fence_after_sync();
        bool ok2 = true;
        if (kStats && FSRC == 2) {
          // both 64-row halves of r^ are written (the buffer holds all 128 rows)
          if (!mbar_wait_bounded(r_full1, (uint32_t)(li & 1), status, kAbort, a.wait_ns)) break;
          tc_fence_after_sync();
          if (rstore) {
            // the tile's r^ image for the later statistics groups' passes
            uint8_t* dst =
                a.rbuf + ((size_t)(((int64_t)cid + li * ncl) * ngrp + grp) * C + rank) * kTcRBytes;
            for (uint32_t q = 0; q < kTcRBytes; q += 16384u) bulk_store(dst + q, sR + q, 16384u);
            bulk_commit();
          }
          ok2 = stats_streamed(li);
          if (rstore) bulk_wait_read();  // before s_done lets the next tile overwrite r^
        } else if (kStats) {
          const bool first = li == 0;  // later tiles add onto whatever the drains left
          if (li > 0) {
            if (!mbar_wait_bounded(drained, ndrain & 1u, status, kAbort, a.wait_ns)) break;
            ndrain++;
            tc_fence_after_sync();
          }
          for (int half = 0; half < 2 && ok2; half++) {
            if (half == 1) {
              mma_commit(r_free);
              ok2 = mbar_wait_bounded(r_full1, (uint32_t)(li & 1), status, kAbort, a.wait_ns);
              if (!ok2) break;
              tc_fence_after_sync();
            }
#pragma unroll
            for (int ks = 0; ks < 4; ks++) {
              const uint64_t ahi = desc_add(dR, 2048u * ks);
              const uint64_t alo = desc_add(dR, 16384u + 2048u * ks);
              const bool acc = !(first && half == 0 && ks == 0);
              const uint32_t kr = 2048u * (uint32_t)(4 * half + ks);  // F rows of this K-step
              const uint64_t fhi = desc_add(dFs, fofs + kr);
              const uint64_t flo = desc_add(dFs, fofs + (uint32_t)nch * kTcChunkBytes + kr);
              mma_bf16(tS, ahi, fhi, idS, acc);
              mma_bf16(tS, ahi, flo, idS, true);
              mma_bf16(tS, alo, fhi, idS, true);
              mma_bf16(tNK, ahi, dOnes, idN, acc);
              mma_bf16(tNK, alo, dOnes, idN, true);
            }
          }
        } else {
          mma_commit(r_free);
          ok2 = mbar_wait_bounded(r_full1, (uint32_t)(li & 1), status, kAbort, a.wait_ns);
        }
        if (!ok2) break;
        mma_commit(s_done);
        if (FSRC == 1) mma_commit(&f_free[li % L.nfb]);
        SCEM_TRACE(li, 11);
      }
      if (rstore) bulk_wait_all();  // the r^ images are in global memory
      // every MMA issued must be complete before tensor memory is released
      mma_commit(final_bar);
      mbar_wait_bounded(final_bar, 0, status, 0u, a.drain_ns);
    }
  } else {
    // ------------------------------------------------------------ compute warps
    const int qd = warp & 3, hf = warp >> 2;
    const int t = tid;                  // 0..255: position in the conversion loop
    const int row = 32 * qd + lane;     // tile row (epilogue), component lane (drains)
    const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
    const int col0 = 64 * hf;           // this thread's 64 component columns
    double ll = 0.0;
    bool ok = true;
    uint32_t ncbar = 0;                 // completed rendezvous on cbar
    const int G = D / 4;

    // bounded rendezvous of the 256 compute threads
    auto rendezvous = [&]() -> bool {
      mbar_arrive(cbar);
      const bool r = __all_sync(0xffffffffu,
                                mbar_wait_bounded(cbar, ncbar & 1u, status, kAbort, a.wait_ns));
      ncbar++;
      return r;
    };

    // Drain component lane `row` into the fp64 slot and zero what was drained.
    // `force`: every accumulator of every component (features not drained
    // since the last forced drain may hold mass even when N_k, drained more
    // often, does not).  Otherwise, for a component with mass in this tile,
    // its precise features only (pmask) and its N_k: those whose fp32 sums
    // would lose too much over several tiles.  Column half 0 also owns the N_k
    // column.
    auto drain = [&](bool force, int64_t li) -> bool {
      const int k = k0 + row;
      float vn[32];
      tmem_ld32(tNK + lane_base, vn);
      const bool due = k < K && (force || (precs[row] != 0 && vn[0] != 0.f));
      if (!rendezvous()) return false;
      if (t == 0) SCEM_TRACE(li, 14);
      if (!__any_sync(0xffffffffu, due)) return true;
      // Fire-and-forget fp64 reductions into the slot: one thread owns each
      // address, so the additions land in program order (deterministic) and
      // the thread does not wait for the old value.
      double* sk = slot + k;
      if (hf == 0) {
        if (due) {
          // (streamed features: N_k is the same in every group's pass; the first adds it)
          if (vn[0] != 0.f && (FSRC != 2 || a.fg0 == 0))
            atomicAdd(sk + (size_t)(2 * D) * K, (double)vn[0]);
#pragma unroll
          for (int j = 0; j < 32; j++) vn[j] = 0.f;
        }
        tmem_st32(tNK + lane_base, vn);
      }
      if (t == 0) SCEM_TRACE(li, 15);
      const uint32_t* pm = a.pmask + (size_t)(due ? k : 0) * (2 * nch);
      // the feature chunks in tensor memory: all, or this pass's statistics group
      const int cbase = FSRC == 2 ? a.fg0 : 0, nchl = FSRC == 2 ? a.nfgc : nch;
      for (int c = 0; c < nchl; c++) {
        const uint32_t mask =
            !due ? 0u : (force ? 0xffffffffu : __ldg(pm + 2 * (cbase + c) + hf));
        if (!__any_sync(0xffffffffu, mask != 0u)) continue;  // nothing of this block is due
        float v[32];
        const uint32_t cc = tS + lane_base + 64u * c + 32u * hf;
        tmem_ld32(cc, v);
        if (mask) {
          const int f0 = 64 * (cbase + c) + 32 * hf;
          const int nf = min(32, 2 * D - f0);  // features of this column block that exist
#pragma unroll
          for (int j = 0; j < 32; j++)
            if ((mask >> j) & 1u) {
              if (j < nf && v[j] != 0.f) atomicAdd(sk + (size_t)(f0 + j) * K, (double)v[j]);
              v[j] = 0.f;
            }
        }
        tmem_st32(cc, v);
      }
      return true;
    };

    // The E-step accumulator of each tile starts from -5/8 Q_k (kTcStartFrac,
    // in W-row-scale units; the rest of the constant is added in the
    // epilogue) rather than from zero, so that its rounding errors cancel.
    // Each thread writes its own row and column half; the stores are waited
    // on before the F-full arrive.
    auto store_start = [&](uint32_t lbuf) {
#pragma unroll
      for (int q = 0; q < 2; q++) {
        float v[32];
#pragma unroll
        for (int j4 = 0; j4 < 8; j4++) {
          const float4 c4 = reinterpret_cast<const float4*>(cis + col0 + 32 * q)[j4];
          v[4 * j4 + 0] = c4.x;
          v[4 * j4 + 1] = c4.y;
          v[4 * j4 + 2] = c4.z;
          v[4 * j4 + 3] = c4.w;
        }
        tmem_st32_nowait(tL + 128u * lbuf + lane_base + (uint32_t)(col0 + 32 * q), v);
      }
    };
    if (my_tiles > 0) {
      store_start(0);
      if (kOverlap) {
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(&f_full2[0]);
      }
    }

    for (int64_t li = 0; li < my_tiles && ok; li++) {
      const int64_t row0 = ((int64_t)cid + li * ncl) * kTcRows;
      if (t == 0) SCEM_TRACE(li, 0);
      // The previous tile's statistics MMAs must be done before its drain and
      // before this tile's r^ reuses their buffer -- and, with one F buffer,
      // before this tile's features overwrite theirs.  With two F buffers the
      // wait moves past the conversion, which then overlaps those MMAs.
      auto wait_prev_stats = [&]() -> bool {
        const bool r = __all_sync(0xffffffffu,
                                  mbar_wait_bounded(s_done, (uint32_t)((li - 1) & 1), status,
                                                    kAbort, a.wait_ns));
        if (t == 0) SCEM_TRACE(li, 1);
        tc_fence_after_sync();
        return r;
      };
      if (rload) {
        // r^ comes from the first group's pass: the previous tile's drain only
        if (li > 0) {
          ok = wait_prev_stats();
          if (ok) ok = drain((li % a.drain_tiles) == 0, li);
          if (!ok) break;
          tc_fence_before_sync();
          mbar_arrive(drained);
        }
        continue;
      }
      if (!FSRC && li > 0 && L.nfb == 1) {
        ok = wait_prev_stats();
        if (!ok) break;
      }
      uint8_t* sFc = sF + (uint32_t)(li % L.nfb) * L.fbytes;  // this tile's F buffer
      const uint32_t tLc = tL + (kOverlap ? 128u * (uint32_t)(li & 1) : 0u);  // its logits
      if (kOverlap && li + 1 < my_tiles) {
        // the next tile's start values into the other logit buffer, read last
        // by the tile before this one
        store_start((uint32_t)((li + 1) & 1));
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(&f_full2[(li + 1) & 1]);
      }
      bool bad = false, wide = false;
      if (!FSRC) {
      // ---- X tile -> F = [x^, x^^2] as fp16 hi/lo in the swizzled layout.
      // The next tile's rows (contiguous in X) are pulled into L2 now, so that
      // its loads meet L2 rather than DRAM latency; up to 16 16-byte loads per
      // thread are in flight before any is converted.
      if (t == 0 && li + 1 < my_tiles) {
        const int64_t nrow0 = row0 + (int64_t)ncl * kTcRows;
        const int64_t nrows = min((int64_t)kTcRows, a.N - nrow0);
        if (nrows > 0)
          prefetch_l2_bulk(reinterpret_cast<const XT*>(a.X) + (size_t)nrow0 * D,
                           (uint32_t)((size_t)nrows * D * sizeof(XT)));
      }
      constexpr int kBatch = 16;
      int nbatch = 0;
      for (int u0 = t; u0 < kTcRows * G; u0 += kTcComputeThreads * kBatch) {
        float xb[kBatch][4];
#pragma unroll
        for (int b = 0; b < kBatch; b++) {
          const int u = u0 + b * kTcComputeThreads;
          const int n = u / G, g = u - n * G;
#pragma unroll
          for (int j = 0; j < 4; j++) xb[b][j] = 0.f;
          if (u < kTcRows * G && row0 + n < a.N)
            load4<XT>(reinterpret_cast<const XT*>(a.X), (size_t)(row0 + n) * D + 4 * g, xb[b]);
        }
        if (t == 0 && nbatch == 0) SCEM_TRACE(li, 12);
#pragma unroll
        for (int b = 0; b < kBatch; b++) {
          const int u = u0 + b * kTcComputeThreads;
          if (u >= kTcRows * G) break;
          const int n = u / G, g = u - n * G;
          float x[4];
          const bool live = row0 + n < a.N;
          const float4 m4 = reinterpret_cast<const float4*>(msm)[g];
          const float4 i4 = reinterpret_cast<const float4*>(iscs)[g];
          const float mv[4] = {m4.x, m4.y, m4.z, m4.w}, iv[4] = {i4.x, i4.y, i4.z, i4.w};
#pragma unroll
          for (int j = 0; j < 4; j++) {
            x[j] = 0.f;
            if (live) {
              if (!isfinite(xb[b][j])) bad = true;
              x[j] = (xb[b][j] - mv[j]) * iv[j];
              if (fabsf(x[j]) > kTcXMax) {
                wide = true;
                x[j] = copysignf(kTcXMax, x[j]);
              }
            }
          }
          uint32_t hx[2], lx[2], hs[2], ls[2];
#pragma unroll
          for (int h = 0; h < 2; h++) {
            const float x0 = x[2 * h], x1 = x[2 * h + 1];
            split_half2(x0, x1, hx[h], lx[h]);
            split_half2(x0 * x0, x1 * x1, hs[h], ls[h]);
          }
          const int f1 = 4 * g, f2 = D + 4 * g;
          const uint32_t o1 = (uint32_t)(f1 >> 6) * kTcChunkBytes + sw128_offset(n, f1 & 63);
          const uint32_t o2 = (uint32_t)(f2 >> 6) * kTcChunkBytes + sw128_offset(n, f2 & 63);
          const uint32_t lo_off = (uint32_t)nch * kTcChunkBytes;
          *reinterpret_cast<uint2*>(sFc + o1) = make_uint2(hx[0], hx[1]);
          *reinterpret_cast<uint2*>(sFc + lo_off + o1) = make_uint2(lx[0], lx[1]);
          *reinterpret_cast<uint2*>(sFc + o2) = make_uint2(hs[0], hs[1]);
          *reinterpret_cast<uint2*>(sFc + lo_off + o2) = make_uint2(ls[0], ls[1]);
        }
        if (t == 0) SCEM_TRACE(li, 13);
        nbatch++;
      }
      }  // !FSRC: conversion
      if (bad) atomicOr(a.status, GMM_DEVFLAG_NONFINITE_X);
      if (wide) atomicOr(a.status, GMM_DEVFLAG_X_RANGE);
      if (!kOverlap) {
        fence_proxy_async_smem();
        tmem_wait_st();  // the accumulator's start values are in place
        tc_fence_before_sync();
        mbar_arrive(f_full);
      }
      if (t == 0) SCEM_TRACE(li, 3);
      if (!kOverlap && li > 0 && (FSRC || L.nfb == 2)) {
        ok = wait_prev_stats();
        if (!ok) break;
      }
      // Drain the previous tiles' statistics while the E-step MMAs run (they
      // write other tensor-memory columns); this tile's statistics MMAs wait
      // for it.
      if (kStats && li > 0) {
        ok = drain((li % a.drain_tiles) == 0, li);
        if (t == 0) SCEM_TRACE(li, 2);
        if (!ok) break;
        tc_fence_before_sync();
        mbar_arrive(drained);
      }

      // ---- epilogue: logits -> row max / sum-exp -> cluster exchange -> r^
      const bool valid = row0 + row < a.N;
      float M = -INFINITY, S = 0.f;
      int win = INT_MAX;  // hard EM: the row's component
      // (max, sum-exp) partials combine as max and the sum rescaled to it;
      // (max, index) partials as max and the lowest index attaining it
      auto combine = [&](const float2 p) {
        if (kHard) {
          const int ix = __float_as_int(p.y);
          if (p.x > M || (p.x == M && ix < win)) win = ix;
          M = fmaxf(M, p.x);
        } else {
          M = fmaxf(M, p.x);
        }
      };
      if ((kStats || MODE == kTcTopm) && ngrp > 1) {
        // The row's partials of every group, from the partial pass over the
        // same rows, combined in group order: the same value in every
        // cluster, so the responsibilities of all groups sum to one.  Read
        // while the E-step MMAs run.
        const float2* pr = a.part + (size_t)(valid ? row0 + row : 0) * ngrp;
        for (uint32_t g2 = 0; g2 < ngrp; g2++) combine(pr[g2]);
        if (!kHard)
          for (uint32_t g2 = 0; g2 < ngrp; g2++) {
            const float2 p = pr[g2];
            if (p.x > -INFINITY) S += p.y * __expf(p.x - M);
          }
      }
      ok = __all_sync(0xffffffffu,
                      kOverlap ? mbar_wait_bounded(&l_full2[li & 1], (uint32_t)((li >> 1) & 1),
                                                   status, kAbort, a.wait_ns)
                               : mbar_wait_bounded(l_full, (uint32_t)(li & 1), status, kAbort,
                                                   a.wait_ns));
      if (!ok) break;
      if (t == 0) SCEM_TRACE(li, 4);
      tc_fence_after_sync();
      float e[64];
      float mx = -INFINITY;
      // first pass (final = false): every column is an accumulator value,
      // scaled to a log-joint; a masked column (a component with exact
      // log-joints) holds that value plus its error bound mg, an upper bound,
      // and counts at the value less mg in the max, a lower bound of the
      // half's best log-joint.  Second pass (final = true): a masked column
      // holds the exact log-joint where the row is near the component (bit
      // set in nb) and is -inf elsewhere.
      auto load_logits = [&](bool final, uint32_t m0, uint32_t m1, uint64_t nb) {
        mx = -INFINITY;
#pragma unroll
        for (int q = 0; q < 2; q++) {
          float v[32];
          tmem_ld32(tLc + lane_base + (uint32_t)(col0 + 32 * q), v);
          const uint32_t mq = q ? m1 : m0;
#pragma unroll
          for (int j = 0; j < 32; j++) {
            const int cidx = col0 + 32 * q + j;
            const bool masked = (mq >> j) & 1u;
            const bool nr = (nb >> (32 * q + j)) & 1ull;
            if (final) {
              e[32 * q + j] = masked ? (nr ? v[j] : -INFINITY) : fmaf(v[j], wscs[cidx], csm[cidx]);
              mx = fmaxf(mx, e[32 * q + j]);
            } else {
              const float l = fmaf(v[j], wscs[cidx], csm[cidx]);
              const float mg = masked ? mgs[cidx] : 0.f;
              e[32 * q + j] = l + mg;
              mx = fmaxf(mx, l - mg);
            }
          }
        }
      };
      const uint32_t sm0 = (uint32_t)shl[kTcComps + 1 + 2 * hf],
                     sm1 = (uint32_t)shl[kTcComps + 2 + 2 * hf];
      load_logits(false, sm0, sm1, 0ull);
      // a lower bound of the row's best log-joint: this half's or, with
      // component groups, the exact row max from the partial pass
      const float mlb = fmaxf(mx, M);
      uint64_t nearb = 0;  // masked columns of this half that the row is near
      if (sm0 | sm1) {
        // Components of this column half with exact log-joints.  A row whose
        // contraction value, plus its error bound, falls 32 nats below a lower
        // bound of its best log-joint (this half's, or with component groups
        // the exact row max from the partial pass) has responsibility below
        // e^-32: its r^ (fp16 of r 2^15) is 0 and it takes no direct-form
        // moments (kTcDirRmin), so it gets -inf.  For the rows near the
        // component the warp computes the log-joint in direct form from X,
        // one row at a time, its lanes over the dimensions, the per-lane sums
        // added in a fixed butterfly order.
        const float floor_l = mlb - 32.f;
        const bool rvalid = row0 + row < a.N;
        if (rvalid) {
          const uint64_t msk = (uint64_t)sm0 | ((uint64_t)sm1 << 32);
#pragma unroll
          for (int j = 0; j < 64; j++)
            if (e[j] > -INFINITY && e[j] >= floor_l) nearb |= 1ull << j;  // e: the upper bound
          nearb &= msk;
        }
        const int* hs = shs + hf * (kTcComps / 2 + 1);
        const int nhs = hs[0];
        const XT* xw = reinterpret_cast<const XT*>(a.X) + (size_t)(row0 + 32 * qd) * D;
        for (int si = 0; si < nhs; si++) {
          const int j = hs[1 + si];
          uint32_t nm = __ballot_sync(0xffffffffu, (nearb >> (j & 63)) & 1ull);
          if (nm == 0u) continue;  // no row of the warp: the column is not read again
          const float* muk = a.mun + (size_t)(k0 + j) * D;
          const float* pk = a.pn + (size_t)(k0 + j) * D;
          float lx = -INFINITY;
          while (nm != 0u) {
            // two rows at a time, so that their loads overlap
            const int s0 = __ffs(nm) - 1;
            nm &= nm - 1u;
            const int s1 = nm != 0u ? __ffs(nm) - 1 : -1;
            if (s1 >= 0) nm &= nm - 1u;
            const XT* x0 = xw + (size_t)s0 * D;
            const XT* x1 = xw + (size_t)(s1 >= 0 ? s1 : s0) * D;
            float q0 = 0.f, q1 = 0.f;
            for (int d = lane; d < D; d += 32) {
              const float mu_d = __ldg(muk + d), p_d = __ldg(pk + d);
              const float e0 = load1<XT>(x0, d) - mu_d, e1 = load1<XT>(x1, d) - mu_d;
              q0 = fmaf(e0 * e0, p_d, q0);
              q1 = fmaf(e1 * e1, p_d, q1);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              q0 += __shfl_xor_sync(0xffffffffu, q0, o);
              q1 += __shfl_xor_sync(0xffffffffu, q1, o);
            }
            if (lane == s0) lx = cxs[j] - 0.5f * q0;
            if (lane == s1) lx = cxs[j] - 0.5f * q1;
          }
          // the exact log-joint (the second load_logits takes it where the row is near)
          tmem_st1(tLc + lane_base + (uint32_t)j, lx);
        }
        load_logits(true, sm0, sm1, nearb);
      }
      if (t == 0) SCEM_TRACE(li, 5);
      float se = 0.f;
      // hard EM: the first column of the thread's largest log-joint, as a
      // component index (INT_MAX when none is finite)
      int own_arg = INT_MAX;
      if (kHard) {
        float best = -INFINITY;
#pragma unroll
        for (int j = 0; j < 64; j++)
          if (e[j] > best) {
            best = e[j];
            own_arg = k0 + col0 + j;
          }
        se = __int_as_float(own_arg);  // exchanged in place of the sum-exp
      } else if (mx > -INFINITY) {
        if (MODE == kTcTopm) {
          // the thread's ncand largest log-joints (ties to the lower index),
          // kept sorted in registers, before they become exponentials
          float cv[kTcCand];
          int ci[kTcCand];
#pragma unroll
          for (int q = 0; q < kTcCand; q++) {
            cv[q] = -INFINITY;
            ci[q] = INT_MAX;
          }
#pragma unroll
          for (int j = 0; j < 64; j++) {
            float v = e[j];
            int ix = k0 + col0 + j;
            if (v > cv[kTcCand - 1]) {
#pragma unroll
              for (int q = 0; q < kTcCand; q++)
                if (v > cv[q]) {  // strictly larger: equal values keep the lower index first
                  const float tv = cv[q];
                  const int ti = ci[q];
                  cv[q] = v;
                  ci[q] = ix;
                  v = tv;
                  ix = ti;
                }
            }
          }
          if (row0 + row < a.N) {
            float2* dst = a.cand + ((size_t)(row0 + row) * (ngrp * (uint32_t)C * 2u) +
                                    ((grp * (uint32_t)C + rank) * 2u + (uint32_t)hf)) *
                                       (size_t)a.ncand;
#pragma unroll
            for (int q = 0; q < kTcCand; q++)
              if (q < a.ncand) dst[q] = make_float2(cv[q], __int_as_float(ci[q]));
          }
        }
#pragma unroll
        for (int j = 0; j < 64; j++) {
          e[j] = __expf(e[j] - mx);
          se += e[j];
        }
      } else {
        // no finite log-joint in this half (dead or padding components, or a
        // row past N): its responsibilities are exactly 0, not -inf * 0
#pragma unroll
        for (int j = 0; j < 64; j++) e[j] = 0.f;
        if (MODE == kTcTopm && row0 + row < a.N) {
          float2* dst = a.cand + ((size_t)(row0 + row) * (ngrp * (uint32_t)C * 2u) +
                                  ((grp * (uint32_t)C + rank) * 2u + (uint32_t)hf)) *
                                     (size_t)a.ncand;
          for (int q = 0; q < a.ncand; q++) dst[q] = make_float2(-INFINITY, __int_as_float(INT_MAX));
        }
      }
      if ((kStats || MODE == kTcTopm) && ngrp > 1) {
        // combined above, before the wait for the E-step
      } else {
        // every (CTA, column half) contributes one (max, sum-exp) partial per row
        const uint32_t par = (uint32_t)(li & 1);
        const uint32_t my_x = smem_u32(&xchg[((par * C + rank) * 2 + hf) * kTcRows + row]);
        for (int r2 = 0; r2 < C; r2++) st_cluster_f32x2(map_to_rank(my_x, r2), mx, se);
        __syncwarp();  // the warp's stores happen before lane 0's release-arrive
        if (lane == 0) {
          // From 4 CTAs up, one cluster-scope fence releases the warp's stores
          // to every CTA's buffer (cumulative over the lanes ordered by the
          // __syncwarp above), then a relaxed arrive on each CTA's barrier
          // (measured: the partial pass of 4-CTA clusters 22 % faster); below,
          // a releasing arrive each (2-CTA clusters were 10 % slower with the fence).
          const uint32_t xb = smem_u32(&xbar[par]);
          if (C >= 4) {
            fence_acq_rel_cluster();
            for (int r2 = 0; r2 < C; r2++) mbar_arrive_cluster_relaxed(map_to_rank(xb, r2));
          } else {
            for (int r2 = 0; r2 < C; r2++) mbar_arrive_cluster(map_to_rank(xb, r2));
          }
        }
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&xbar[par], (uint32_t)((li >> 1) & 1),
                                                       status, kAbort, a.wait_ns, true));
        if (!ok) break;
        if (t == 0) SCEM_TRACE(li, 6);
        for (int j = 0; j < 2 * C; j++) combine(xchg[(par * C * 2 + j) * kTcRows + row]);
        if (!kHard)
          for (int j = 0; j < 2 * C; j++) {
            const float2 p = xchg[(par * C * 2 + j) * kTcRows + row];
            if (p.x > -INFINITY) S += p.y * __expf(p.x - M);
          }
        if (kPartial && valid && rank == 0 && hf == 0)
          a.part[(size_t)(row0 + row) * ngrp + grp] =
              make_float2(M, kHard ? __int_as_float(win) : S);
      }
      // soft: the row's log-sum-exp; hard: its largest log-joint
      const float lse = kHard ? M : M + __logf(S);
      if (MODE == kTcTopm && valid && rank == 0 && hf == 0 && grp == 0)
        a.rowst[row0 + row] = make_float2(M, S);
      if (!kPartial && MODE != kTcTopm && valid && rank == 0 && hf == 0 && grp == 0 &&
          (FSRC != 2 || a.fg0 == 0)) {
        ll += (double)lse;
        if (kHard && a.labels) a.labels[row0 + row] = win < K ? win : -1;
      }
      float scale = (valid && mx > -INFINITY) ? __expf(mx - lse) * kTcRScale : 0.f;
      if (kHard) {
        // one-hot: exactly 2^15 in the winning column, zero elsewhere
#pragma unroll
        for (int j = 0; j < 64; j++) e[j] = (k0 + col0 + j == win) ? 1.f : 0.f;
        scale = valid ? kTcRScale : 0.f;
      }
      const int hr = row >> 6, rr = row & 63;  // which 64-row half of r^, row within it
      uint64_t rbits = 0;  // the thread's columns whose r exceeds kTcDirRmin
      if (kStats) {
        if (FSRC != 2 && hr == 1) {
          // the first half's MMAs must be done with the buffer
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(r_free, (uint32_t)(li & 1), status,
                                                         kAbort, a.wait_ns));
          if (!ok) break;
        }
#pragma unroll
        for (int q8 = 0; q8 < 8; q8++) {
          uint4 ph4, pl4;
          split_half2(e[8 * q8 + 0] * scale, e[8 * q8 + 1] * scale, ph4.x, pl4.x);
          split_half2(e[8 * q8 + 2] * scale, e[8 * q8 + 3] * scale, ph4.y, pl4.y);
          split_half2(e[8 * q8 + 4] * scale, e[8 * q8 + 5] * scale, ph4.z, pl4.z);
          split_half2(e[8 * q8 + 6] * scale, e[8 * q8 + 7] * scale, ph4.w, pl4.w);
          const uint32_t off = (FSRC == 2 ? 32768u * (uint32_t)hr : 0u) + (uint32_t)hf * 8192u +
                               (uint32_t)rr * 128u + ((((uint32_t)q8) ^ ((uint32_t)rr & 7u)) << 4);
          *reinterpret_cast<uint4*>(sR + off) = ph4;
          *reinterpret_cast<uint4*>(sR + 16384u + off) = pl4;
        }
        if (shl[0] > 0) {
#pragma unroll
          for (int j = 0; j < 64; j++)
            if (e[j] * scale > kTcDirRmin * kTcRScale) rbits |= 1ull << j;
        }
        fence_proxy_async_smem();
      }
      tc_fence_before_sync();
      mbar_arrive(hr == 0 ? r_full : r_full1);
      if (t == 0) SCEM_TRACE(li, 7);
      // Moments of split dimensions in direct form, about the input means, in
      // data units from X (no cancellation however narrow the dimension),
      // while the statistics MMAs run.  Only rows whose responsibility exceeds
      // kTcDirRmin contribute: the few near the component.  (X, not F: F may
      // already hold the next tile once the statistics MMAs are done.)  Each
      // row's terms are rounded to the fixed-point unit kTcDirScale; a warp
      // takes one component at a time, its lanes over 32 of the component's
      // dimensions, sums the terms of its active rows as 64-bit integers and
      // adds the sums to the shared fixed-point area with one coalesced
      // atomic per word.  Integer sums do not depend on the order in which
      // rows, warps and clusters add them.
      if (kStats && shl[0] > 0 && (FSRC != 2 || a.fg0 == 0)) {
        // the components of this half with direct dimensions that some row
        // of the warp needs (a warp-uniform set: the tensor-memory load below
        // is a warp-collective .sync.aligned instruction)
        const uint64_t exact = (uint64_t)sm0 | ((uint64_t)sm1 << 32);
        const uint64_t direct =
            (uint64_t)(uint32_t)ndc[kTcComps + 2 * hf] |
            ((uint64_t)(uint32_t)ndc[kTcComps + 2 * hf + 1] << 32);
        const uint64_t need =
            (((uint64_t)__reduce_or_sync(0xffffffffu, (uint32_t)(rbits >> 32)) << 32) |
             (uint64_t)__reduce_or_sync(0xffffffffu, (uint32_t)rbits)) & direct;
        for (uint64_t todo = need; todo != 0ull; todo &= todo - 1ull) {
          const int jj = __ffsll((long long)todo) - 1, j = col0 + jj;
          const int nd = ndc[j];
          // the log-joint: exact in tensor memory for a component with exact
          // log-joints where the row is near it (-inf elsewhere), the raw
          // accumulator (scaled as the epilogue scales it) otherwise
          const float v0 = tmem_ld1(tLc + lane_base + (uint32_t)j);
          const float l = !((exact >> jj) & 1ull) ? fmaf(v0, wscs[j], csm[j])
                          : ((nearb >> jj) & 1ull) ? v0 : -INFINITY;
          const double r = !(valid && l > -INFINITY) ? 0.0
                           : kHard ? (k0 + j == win ? 1.0 : 0.0)
                                   : (double)__expf(l - lse);
          const uint32_t active = __ballot_sync(0xffffffffu, r > (double)kTcDirRmin);
          if (active == 0u) continue;
          const size_t base = (size_t)(k0 + j) * D;
          unsigned long long* q = a.dirq + (size_t)(k0 + j) * (4 * D);
          for (int i0 = 0; i0 < nd; i0 += 32) {
            const int i = i0 + lane;
            const bool has = i < nd;
            const int d = has ? min((int)a.perm[base + i], D - 1) : 0;
            const double mu_i = has ? (double)a.muh[base + i] : 0.0;
            const double isd = has ? sqrt((double)a.ph[base + i]) : 0.0;  // 1/sigma
            long long sa = 0, sb = 0;
            for (uint32_t m = active; m != 0u; m &= m - 1u) {
              const int src = __ffs(m) - 1;
              const double rs = __shfl_sync(0xffffffffu, r, src);
              if (has) {
                const XT* xs = reinterpret_cast<const XT*>(a.X) +
                               (size_t)(row0 + 32 * qd + src) * D;  // a valid row: r > 0
                const double u = ((double)load1<XT>(xs, d) - mu_i) * isd;
                const double ru = rs * u * kTcDirScale;
                sa += __double2ll_rn(ru);
                sb += __double2ll_rn(ru * u);
              }
            }
            if (has) {
              atomicAdd(q + i, (unsigned long long)(sa >> 32));
              atomicAdd(q + D + i, (unsigned long long)(sa & 0xffffffffll));
              atomicAdd(q + 2 * D + i, (unsigned long long)(sb >> 32));
              atomicAdd(q + 3 * D + i, (unsigned long long)(sb & 0xffffffffll));
            }
          }
        }
      }
      if (!kOverlap && li + 1 < my_tiles) store_start(0);  // L is no longer read in this tile
    }
    if (!kOverlap && ok && my_tiles > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(s_done, (uint32_t)((my_tiles - 1) & 1),
                                                     status, kAbort, a.wait_ns));
      tc_fence_after_sync();
      if (ok && kStats) ok = drain(true, my_tiles);
    }
    // LL of this CTA's rows (rank 0 of each cluster, column half 0): fixed-order sum
    ll = warp_sum(ll);
    double* red = reinterpret_cast<double*>(sR);  // r^ is no longer read by any MMA
    __syncwarp();
    if (lane == 0) red[warp] = ok ? ll : 0.0;
    const bool met = rendezvous();
    if (!kPartial && MODE != kTcTopm && t == 0 && rank == 0) {
      double s = 0.0;
      for (int w = 0; w < 8; w++) s += red[w];
      slot[ll_index] = (a.accumulate ? slot[ll_index] : 0.0) + ((ok && met) ? s : 0.0);
    }
  }

  // ---------------------------------------------------------------- teardown
  if (warp < kTcMmaWarp) tmem_wait_st();
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
  cluster_sync();
}

// ---------------------------------------------------------------------------
// Prep for the tensor-core pass, per dimension:
//   m_d = sum_k pi_k mu_kd / sum_k pi_k                  (centring, fp64)
//   v_d = sum_k pi_k (var_kd + mu_kd^2) / sum_k pi_k - m_d^2   (mixture variance)
//   s_d = 2^(round(log2 sqrt(v_d)) + 1)                  (exact power-of-two scale)
// ---------------------------------------------------------------------------
// One block of 256 threads per dimension: thread t sums components t, t + 256,
// ... in order, then a fixed tree combines the threads (deterministic).
__global__ void __launch_bounds__(256) tc_center_kernel(int D, int K, const float* __restrict__ w,
                                                        const float* __restrict__ mu,
                                                        const float* __restrict__ var,
                                                        float* __restrict__ m_out,
                                                        float* __restrict__ isc_out,
                                                        float* __restrict__ sc_out) {
  __shared__ double red[3][256];
  const int d = blockIdx.x;
  double s = 0.0, s2 = 0.0, sw = 0.0;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const double wk = (double)w[k];
    if (wk > 0.0) {
      const double mk = (double)mu[(size_t)k * D + d];
      s += wk * mk;
      s2 += wk * ((double)var[(size_t)k * D + d] + mk * mk);
      sw += wk;
    }
  }
  red[0][threadIdx.x] = s;
  red[1][threadIdx.x] = s2;
  red[2][threadIdx.x] = sw;
  __syncthreads();
  for (int h = 128; h > 0; h >>= 1) {
    if ((int)threadIdx.x < h)
      for (int q = 0; q < 3; q++) red[q][threadIdx.x] += red[q][threadIdx.x + h];
    __syncthreads();
  }
  if (threadIdx.x != 0) return;
  s = red[0][0];
  s2 = red[1][0];
  sw = red[2][0];
  const double m = sw > 0.0 ? s / sw : 0.0;
  const double v = sw > 0.0 ? s2 / sw - m * m : 0.0;
  int e = 0;
  if (v > 0.0 && isfinite(v)) {
    e = (int)lrint(0.5 * log2(v)) + 1;
    e = max(-60, min(60, e));
  }
  m_out[d] = (float)m;
  isc_out[d] = ldexpf(1.0f, -e);
  sc_out[d] = ldexpf(1.0f, e);
}

inline size_t tc_prep_smem_bytes(int D, int Fpad) {
  return (size_t)(4 * D + 2 * Fpad) * sizeof(double);
}

// One block of 128 threads per (padded) component, looping over the dimensions.
//
// Exact log-joints.  The expanded form's fp32 error grows with
// kappa_k = sum_d (mu^_kd^2 + 1)/var^_kd.  When kappa_k exceeds kTcSharpKappa (a
// component collapsed onto a few points in some dimensions), or kTcSmallKappa
// for a component expecting fewer than kTcSmallPoints points, the contraction's
// log-joint serves only to find the rows near the component: it is within
// mg_k = 1 + 2^-14 kappa_k nats of the exact one (the accumulated fp32 error is
// about 4e-8 kappa_k; the bound allows well over a hundred times that), and a
// row whose contraction value lies more than 80 + mg_k nats below the row's
// best lower bound has responsibility 0.  For the others the kernel computes
// log pi_k - 1/2 sum_d [log(2 pi var_kd) + (x_d - mu_kd)^2/var_kd] in data units
// on the CUDA cores (cx_k the constant part; mun, pn the tables).  nsplit_k > 0
// marks these components (the count of leading dimensions, by kappa_kd, that
// bring the rest below the threshold).  Independently, the leading ndir_k
// dimensions with kappa_kd > kTcDirectKappa take their moments in direct form.
//
// W = [mu^/var^, -1/(2 var^)] over all dimensions, scaled by a power of two
// 2^-g_k so its largest entry lies in [2^13, 2^14), split into fp16 hi/lo rows
// of Fpad features (padding rows and features zero).
//
// The expanded-form constant c_k = log pi_k - (1/2) sum_d log(2 pi var_kd)
// - (1/2) sum_d mu^_kd^2 / var^_kd is corrected for the part of W that
// the fp16 hi/lo split drops: the MMA sums F (W_hi + W_lo) 2^g, short of F W 2^g
// by F dW 2^g with dW = W 2^-g - W_hi - W_lo, known exactly here.  For the
// points the component explains F is near its expectation E[F] = [mu^,
// mu^^2 + var^], so 2^g E[F] . dW is added to c_k: that removes the split's
// systematic error on those points (what remains is (F - E[F]) . dW, of either
// sign from point to point).  The accumulator starts from ci_k = kTcStartFrac
// sum_d mu^^2/var^ (fp32, in 2^g units); the fp32 remainder c_k - 2^g ci_k is
// added after the MMAs.
//
// Tables for the direct-form moments, in perm order: mu and 1/var in data units.
__global__ void __launch_bounds__(128) tc_prep_w_kernel(
    int64_t N, int D, int K, int Fpad, const float* __restrict__ w, const float* __restrict__ mu,
    const float* __restrict__ var, const float* __restrict__ m, const float* __restrict__ sc,
    __half* __restrict__ whi, __half* __restrict__ wlo, float* __restrict__ c_out,
    float* __restrict__ wsc_out, int* __restrict__ ndir_out, int* __restrict__ nsplit_out,
    float* __restrict__ muh, float* __restrict__ ph, int* __restrict__ precise_out,
    float* __restrict__ ci_out, float* __restrict__ cx_out, float* __restrict__ mg_out,
    uint16_t* __restrict__ perm_out, float* __restrict__ mun_out, float* __restrict__ pn_out,
    uint32_t* __restrict__ pmask_out, uint16_t* __restrict__ rank_out,
    unsigned long long* __restrict__ dirq, unsigned int* status) {
  // dynamic shared memory (tc_prep_smem_bytes): per dimension mu^, var^, kappa_kd and
  // kappa sorted; per feature W and E[F] (doubles)
  extern __shared__ double prep_sm[];
  double* mh_s = prep_sm;
  double* vh_s = mh_s + D;
  double* kd_s = vh_s + D;
  double* ksort = kd_s + D;
  double* wv = ksort + D;    // Fpad
  double* ef = wv + Fpad;    // Fpad: E[F] under the component
  __shared__ double red[4][4];
  __shared__ int ns_s, nd_s;
  const int k = blockIdx.x;
  const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
  const float wk = k < K ? w[k] : 0.f;
  // the fused pass adds this component's split-dimension moments onto zero
  for (int q = threadIdx.x; q < 4 * D; q += blockDim.x) dirq[(size_t)k * (4 * D) + q] = 0ull;
  const bool live = k < K && wk > 0.f;
  auto block_sum = [&](double v) -> double {
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) red[0][wp] = v;
    __syncthreads();
    return red[0][0] + red[0][1] + red[0][2] + red[0][3];
  };
  auto block_max = [&](double v) -> double {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if (lane == 0) red[0][wp] = v;
    __syncthreads();
    return fmax(fmax(red[0][0], red[0][1]), fmax(red[0][2], red[0][3]));
  };

  // ---- pass 1: per dimension
  double s_log = 0.0, kap = 0.0, rho = 0.0;
  bool bad = false;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    double mh = 0.0, vh = 1.0, kd = 0.0;
    if (k < K) {
      const double sd = (double)sc[d];
      const double vr = (double)var[(size_t)k * D + d];
      vh = vr / (sd * sd);
      mh = ((double)mu[(size_t)k * D + d] - (double)m[d]) / sd;
      kd = (mh * mh + 1.0) / vh;
      s_log += log(2.0 * M_PI * vr);
      kap += kd;
      if (live) rho = fmax(rho, mh * mh / vh);
      if (!isfinite(mu[(size_t)k * D + d]) || !(vr > 0.0) || !isfinite(vr)) bad = true;
    }
    mh_s[d] = mh;
    vh_s[d] = vh;
    mun_out[(size_t)k * D + d] = k < K ? mu[(size_t)k * D + d] : 0.f;
    pn_out[(size_t)k * D + d] = k < K ? (float)(1.0 / (double)var[(size_t)k * D + d]) : 0.f;
    kd_s[d] = kd >= 0.0 ? fmin(kd, 1e300) : 0.0;  // NaN -> 0: the ranks stay a permutation
  }
  const double S_log = block_sum(s_log);
  const double Kap = block_sum(kap);
  const double Rho = block_max(rho);
  const bool small = (double)wk * (double)N < kTcSmallPoints;
  // the fp32 error grows with the number of accumulation steps, 2D / 16 per
  // operand pair: the thresholds hold for D <= 128 and scale as 128 / D beyond
  const double thr = (small ? kTcSmallKappa : kTcSharpKappa) * fmin(1.0, 128.0 / (double)D);
  const bool sharp = live && Kap > thr;

  // ---- dimensions by decreasing kappa_kd (ties to the lower index)
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    const double key = kd_s[d];
    int r = 0;
    for (int e2 = 0; e2 < D; e2++) {
      const double o = kd_s[e2];
      r += (o > key || (o == key && e2 < d)) ? 1 : 0;
    }
    ksort[r] = key;
    rank_out[(size_t)k * D + d] = (uint16_t)r;
    const size_t o = (size_t)k * D + r;
    perm_out[o] = (uint16_t)d;
    muh[o] = k < K ? mu[(size_t)k * D + d] : 0.f;
    ph[o] = k < K ? (float)(1.0 / (double)var[(size_t)k * D + d]) : 0.f;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int ns = 0;
    if (sharp) {
      double rem = Kap;
      while (ns < D && rem > thr) rem -= ksort[ns++];
    }
    ns_s = ns;
    // the leading dimensions whose moments are taken in direct form
    int nd = 0;
    if (live)
      while (nd < D && ksort[nd] > kTcDirectKappa) nd++;
    nd_s = nd;
  }
  __syncthreads();
  const int ns = ns_s;

  // ---- pass 2: the contraction's features
  double s_q = 0.0, amax = 0.0;
  for (int f = threadIdx.x; f < Fpad; f += blockDim.x) {
    double v = 0.0, e = 0.0;
    if (k < K && f < 2 * D) {
      const int d = f < D ? f : f - D;
      const double mh = mh_s[d], vh = vh_s[d];
      if (f < D) {
        v = mh / vh;
        e = mh;
        s_q += mh * mh / vh;
      } else {
        v = -0.5 / vh;
        e = mh * mh + vh;
      }
    }
    wv[f] = v;
    ef[f] = e;
    amax = fmax(amax, fabs(v));
  }
  const double S_q = block_sum(s_q);
  const double Amax = block_max(amax);
  // Precise features: both features of a dimension with mu^^2/var^ > kTcRhoPrecise
  // (the variance S2/N - (S1/N)^2 magnifies their fp32 rounding by that ratio),
  // every feature of a component expecting fewer than kTcSmallPoints points --
  // except the dimensions whose moments are taken in direct form (the first
  // nd in perm order), whose tensor-core sums are not used.
  for (int f = threadIdx.x; f < Fpad; f += blockDim.x) {  // warp w: features 32w.. of each 128
    bool pf = false;
    if (live && f < 2 * D) {
      const int d = f < D ? f : f - D;
      pf = (small || mh_s[d] * mh_s[d] / vh_s[d] > kTcRhoPrecise) &&
           (int)rank_out[(size_t)k * D + d] >= nd_s;
    }
    const uint32_t word = __ballot_sync(0xffffffffu, pf);
    if (lane == 0) pmask_out[(size_t)k * (Fpad / 32) + f / 32] = word;
  }
  int ex = 0;
  if (Amax > 0.0 && isfinite(Amax)) frexp(Amax, &ex);
  const int g = Amax > 0.0 ? ex - 14 : 0;
  double dsplit = 0.0;  // E[F] . dW in 2^g units
  for (int f = threadIdx.x; f < Fpad; f += blockDim.x) {
    const double svd = ldexp(wv[f], -g);
    const float sv = (float)svd;
    const __half h = __float2half_rn(sv);
    const __half l = __float2half_rn(sv - __half2float(h));
    whi[(size_t)k * Fpad + f] = h;
    wlo[(size_t)k * Fpad + f] = l;
    dsplit += ef[f] * (svd - (double)__half2float(h) - (double)__half2float(l));
  }
  const double Dsplit = block_sum(dsplit);
  if (threadIdx.x == 0) {
    if (k < K && (!isfinite(wk) || !(wk >= 0.f))) bad = true;
    const double lw = live ? log((double)wk) : 0.0;
    const double cfull = lw - 0.5 * (S_log + S_q) + ldexp(Dsplit, g);
    const float cstart = live ? (float)ldexp(kTcStartFrac * S_q, -g) : 0.f;
    ci_out[k] = cstart;
    c_out[k] = live ? (float)(cfull - ldexp((double)cstart, g)) : -INFINITY;
    cx_out[k] = live ? (float)(lw - 0.5 * S_log) : -INFINITY;
    mg_out[k] = ns > 0 ? (float)(1.0 + ldexp(Kap, -14)) : 0.f;
    wsc_out[k] = ldexpf(1.0f, g);
    ndir_out[k] = nd_s;
    nsplit_out[k] = ns;
    precise_out[k] = live && (Rho > kTcRhoPrecise || small) ? 1 : 0;  // some pmask bit set
  }
  if (bad) atomicOr(status, GMM_DEVFLAG_BAD_PARAMS);
}

// Value of a fixed-point pair of sums (see kTcDirScale), in units of 2^-32.
__device__ __forceinline__ double fixed_value(unsigned long long hi, unsigned long long lo) {
  return (double)(long long)hi * kTcDirScale + (double)lo;
}

// Fixed-order fp64 sum of the per-cluster slots into the canonical
// statistics buffer [ N_k | A | B | LL ] (component-major, moments about the
// input means mu, data units).  The slots hold N' = 2^15 N_k and
// S1' = 2^15 sum r x^, S2' = 2^15 sum r x^^2 with x^ = (x - m)/s, so with
// dm = mu - m:  A = s S1 - dm N,  B = s^2 S2 - 2 s dm S1 + dm^2 N.  A
// dimension with direct-form moments (perm position below ndir_k) takes A and
// B from the fixed-point sums instead, scaled back by sigma = 1/sqrt(ph) with the same
// stored ph the fused pass divided by.
__global__ void __launch_bounds__(256) tc_reduce_stats_kernel(
    int D, int K, int Kpad, const float* __restrict__ m, const float* __restrict__ sc,
    const float* __restrict__ mu, const uint16_t* __restrict__ rank,
    const int* __restrict__ ndir, const float* __restrict__ ph,
    const unsigned long long* __restrict__ dirq, const double* __restrict__ slots,
    size_t slot_stride, int nslots, int G, int group_comps, double* __restrict__ stats) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t KD = (size_t)K * D;
  if (i == 0) {
    double ll = 0.0;
    for (int p = 0; p < nslots; p++) ll += slots[(size_t)p * slot_stride + (size_t)(2 * D + 1) * K];
    stats[K + 2 * KD] = ll;
  }
  if (i >= KD) return;
  const int d = (int)(i / K), k = (int)(i - (size_t)d * K);
  double nks = 0.0, s1 = 0.0, s2 = 0.0;
  // the slots of the clusters that served component k's group: g, g + G, ...
  for (int p = k / group_comps; p < nslots; p += G) {
    const double* s = slots + (size_t)p * slot_stride;
    nks += s[(size_t)(2 * D) * K + k];
    s1 += s[(size_t)d * K + k];
    s2 += s[(size_t)(D + d) * K + k];
  }
  const double inv = 1.0 / (double)kTcRScale;
  const double n = nks * inv, S1 = s1 * inv, S2 = s2 * inv;
  const double sd = (double)sc[d];
  const double dm = (double)mu[(size_t)k * D + d] - (double)m[d];
  if (d == 0) stats[k] = n;
  const int r = rank[(size_t)k * D + d];
  if (r < ndir[k]) {
    const double p = (double)ph[(size_t)k * D + r];  // 1/var, perm order
    const unsigned long long* q = dirq + (size_t)k * (4 * D);
    const double a1 = fixed_value(q[r], q[D + r]);
    const double b1 = fixed_value(q[2 * D + r], q[3 * D + r]);
    stats[K + (size_t)k * D + d] = a1 / kTcDirScale / sqrt(p);
    stats[K + KD + (size_t)k * D + d] = b1 / kTcDirScale / p;
    return;
  }
  stats[K + (size_t)k * D + d] = sd * S1 - dm * n;
  stats[K + KD + (size_t)k * D + d] = sd * sd * S2 - 2.0 * sd * dm * S1 + dm * dm * n;
}

// Features of a chunk of rows for the two-pass form: the same x^ = (x - m)/s,
// clamp and fp16 hi/lo split as the fused kernel's own conversion, written
// row-major [rows x Fpad] (x^ in features 0..D-1, x^^2 in D..2D-1, zeros
// after), to be read back tile by tile by TMA in the 128-byte-swizzled
// shared-memory layout.  Raises the same status bits.
template <typename XT>
__global__ void __launch_bounds__(256) tc_convert_kernel(
    const XT* __restrict__ X, int64_t rows, int D, int Fpad, const float* __restrict__ m,
    const float* __restrict__ isc, __half* __restrict__ fhi, __half* __restrict__ flo,
    unsigned int* status) {
  const int G4 = D / 4;
  const int64_t items = rows * G4;
  bool bad = false, wide = false;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < items;
       u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = u / G4;
    const int g = (int)(u - n * G4);
    float xv[4];
    load4<XT>(X, (size_t)n * D + 4 * g, xv);
    float x[4];
#pragma unroll
    for (int j = 0; j < 4; j++) {
      if (!isfinite(xv[j])) bad = true;
      x[j] = (xv[j] - m[4 * g + j]) * isc[4 * g + j];
      if (fabsf(x[j]) > kTcXMax) {
        wide = true;
        x[j] = copysignf(kTcXMax, x[j]);
      }
    }
    uint32_t hx[2], lx[2], hs[2], ls[2];
#pragma unroll
    for (int h = 0; h < 2; h++) {
      split_half2(x[2 * h], x[2 * h + 1], hx[h], lx[h]);
      split_half2(x[2 * h] * x[2 * h], x[2 * h + 1] * x[2 * h + 1], hs[h], ls[h]);
    }
    const size_t o1 = (size_t)n * Fpad + 4 * g, o2 = o1 + D;
    *reinterpret_cast<uint2*>(fhi + o1) = make_uint2(hx[0], hx[1]);
    *reinterpret_cast<uint2*>(flo + o1) = make_uint2(lx[0], lx[1]);
    *reinterpret_cast<uint2*>(fhi + o2) = make_uint2(hs[0], hs[1]);
    *reinterpret_cast<uint2*>(flo + o2) = make_uint2(ls[0], ls[1]);
  }
  // padding features read as zero in every MMA
  const int P4 = (Fpad - 2 * D) / 4;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < rows * P4;
       u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = u / P4;
    const size_t o = (size_t)n * Fpad + 2 * D + 4 * (u - n * P4);
    *reinterpret_cast<uint2*>(fhi + o) = make_uint2(0u, 0u);
    *reinterpret_cast<uint2*>(flo + o) = make_uint2(0u, 0u);
  }
  if (bad) atomicOr(status, GMM_DEVFLAG_NONFINITE_X);
  if (wide) atomicOr(status, GMM_DEVFLAG_X_RANGE);
}

// Top-m from the fused pass's candidates, one thread per row.  The row's
// P = G C 2 candidate lists (each sorted by tensor-core log-joint, ties to the
// lower index) are merged into its nc best.  Their log-joints are recomputed
// in direct form in fp32, l_k = c0_k - 1/2 sum_d (x_d - mu_kd)^2 iv_kd with
// c0_k = log pi_k - 1/2 sum_d log(2 pi var_kd) and iv = 1/var, and exchanged
// for their tensor-core terms in the row's sum-exp (the candidates carry
// almost all of a row's mass, so the normalisation comes out as precise as
// the direct form).  r_k = exp(l_k - lse); the candidates are ordered by r,
// descending, equal r to the lower index, and the first m written.  A row
// with fewer than m finite candidates is completed, r = 0, by the lowest
// indices not yet taken (the same order the definition gives).
template <typename XT>
__global__ void __launch_bounds__(128) tc_topm_refine_kernel(
    const XT* __restrict__ X, int64_t rows, int D, int K, int P, int nc, int m,
    const float2* __restrict__ cand, const float2* __restrict__ rowst,
    const float* __restrict__ mu, const float* __restrict__ iv, const float* __restrict__ c0,
    int32_t* __restrict__ idx_out, float* __restrict__ resp_out) {
  const int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= rows) return;
  float bv[kTcCand], bl[kTcCand];
  int bi[kTcCand];
#pragma unroll
  for (int q = 0; q < kTcCand; q++) {
    bv[q] = -INFINITY;
    bi[q] = INT_MAX;
  }
  const float2* cr = cand + (size_t)n * P * nc;
  for (int i = 0; i < P * nc; i++) {
    const float2 c = cr[i];
    float v = c.x;
    int ix = __float_as_int(c.y);
    if (!(v > -INFINITY)) continue;
    // insert into the sorted best nc: (value desc, index asc)
#pragma unroll
    for (int q = 0; q < kTcCand; q++)
      if (q < nc && (v > bv[q] || (v == bv[q] && ix < bi[q]))) {
        const float tv = bv[q];
        const int ti = bi[q];
        bv[q] = v;
        bi[q] = ix;
        v = tv;
        ix = ti;
      }
  }
  const float2 st = rowst[n];
  const float M = st.x;
  float S = st.y;
  const XT* xr = X + (size_t)n * D;
#pragma unroll
  for (int q = 0; q < kTcCand; q++) {
    bl[q] = -INFINITY;
    if (q < nc && bi[q] < K) {
      const int k = bi[q];
      const float* mk = mu + (size_t)k * D;
      const float* ik = iv + (size_t)k * D;
      float qd = 0.f;
      for (int d = 0; d < D; d++) {
        const float e = load1<XT>(xr, d) - mk[d];
        qd = fmaf(e * e, ik[d], qd);
      }
      bl[q] = c0[k] - 0.5f * qd;
      S += __expf(bl[q] - M) - __expf(bv[q] - M);
    }
  }
  const float lse = M + __logf(S);
  float r[kTcCand];
#pragma unroll
  for (int q = 0; q < kTcCand; q++) r[q] = bl[q] > -INFINITY ? __expf(bl[q] - lse) : 0.f;
  // order the candidates by (r desc, index asc): insertion sort of nc <= 8
#pragma unroll
  for (int a1 = 1; a1 < kTcCand; a1++)
#pragma unroll
    for (int b1 = a1; b1 > 0; b1--)
      if (b1 < nc && (r[b1] > r[b1 - 1] || (r[b1] == r[b1 - 1] && bi[b1] < bi[b1 - 1]))) {
        const float tr = r[b1];
        r[b1] = r[b1 - 1];
        r[b1 - 1] = tr;
        const int ti = bi[b1];
        bi[b1] = bi[b1 - 1];
        bi[b1 - 1] = ti;
      }
  int32_t* io = idx_out + (size_t)n * m;
  float* ro = resp_out + (size_t)n * m;
  int j = 0;
  for (int q = 0; q < nc && j < m; q++)
    if (bi[q] < K && r[q] > 0.f) {
      io[j] = bi[q];
      ro[j] = r[q];
      j++;
    }
  // zero responsibilities: the lowest indices not taken yet
  for (int k = 0; j < m && k < K; k++) {
    bool taken = false;
    for (int q = 0; q < j; q++) taken |= io[q] == k;
    if (!taken) {
      io[j] = k;
      ro[j] = 0.f;
      j++;
    }
  }
}

// 1/var and c0_k = log pi_k - 1/2 sum_d log(2 pi var_kd) (-inf for pi_k = 0)
// for the refinement, one block per component.
__global__ void __launch_bounds__(128) tc_topm_prep_kernel(int D, const float* __restrict__ w,
                                                           const float* __restrict__ var,
                                                           float* __restrict__ iv,
                                                           float* __restrict__ c0) {
  __shared__ double red[128];
  const int k = blockIdx.x;
  double s = 0.0;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    const float v = var[(size_t)k * D + d];
    iv[(size_t)k * D + d] = 1.0f / v;
    s += log(2.0 * M_PI * (double)v);
  }
  red[threadIdx.x] = s;
  __syncthreads();
  for (int h = 64; h > 0; h >>= 1) {
    if ((int)threadIdx.x < h) red[threadIdx.x] += red[threadIdx.x + h];
    __syncthreads();
  }
  if (threadIdx.x == 0) c0[k] = w[k] > 0.f ? (float)(log((double)w[k]) - 0.5 * red[0]) : -INFINITY;
}

constexpr int kTcLseBlocks = 128;

// Log-likelihood of a chunk from the groups' partials: each row's log-sum-exp
// combined exactly as the statistics pass combines it, summed in a fixed
// order -- rows [b*per, (b+1)*per) by block b, strided by thread, then a
// fixed tree -- into out[b].
__global__ void __launch_bounds__(256) tc_part_loglik_kernel(const float2* __restrict__ part,
                                                             int64_t rows, int G,
                                                             double* __restrict__ out) {
  __shared__ double red[256];
  const int64_t per = (rows + gridDim.x - 1) / gridDim.x;
  const int64_t lo = (int64_t)blockIdx.x * per, hi = min(rows, lo + per);
  double s = 0.0;
  for (int64_t n = lo + threadIdx.x; n < hi; n += blockDim.x) {
    const float2* pr = part + (size_t)n * G;
    float M = -INFINITY, S = 0.f;
    for (int g = 0; g < G; g++) M = fmaxf(M, pr[g].x);
    for (int g = 0; g < G; g++) {
      const float2 p = pr[g];
      if (p.x > -INFINITY) S += p.y * __expf(p.x - M);
    }
    s += (double)(M + __logf(S));
  }
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) out[blockIdx.x] = red[0];
}

// *acc (+)= sum of the kTcLseBlocks block sums, in block order.
__global__ void tc_sum_blocks_kernel(const double* __restrict__ blocks, int first,
                                     double* __restrict__ acc) {
  double s = 0.0;
  for (int b = 0; b < kTcLseBlocks; b++) s += blocks[b];
  *acc = (first ? 0.0 : *acc) + s;
}

__global__ void tc_reduce_loglik_kernel(int D, int K, const double* __restrict__ slots,
                                        size_t slot_stride, int nslots,
                                        double* __restrict__ loglik) {
  const size_t ll_index = (size_t)(2 * D + 1) * K;
  double ll = 0.0;
  for (int p = 0; p < nslots; p++) ll += slots[(size_t)p * slot_stride + ll_index];
  *loglik = ll;
}

}  // namespace scem
