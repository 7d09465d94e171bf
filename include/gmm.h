/*
 * gmm.h -- C ABI of the B200 (sm_100a) fused EM library for diagonal-covariance
 * Gaussian mixtures.
 *
 * Method: "Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering"
 * (abstract; review page sections 1 and 3).  One EM iteration is one pass over
 * the data in tiles: each tile's E-step log-densities, its per-point
 * log-sum-exp normalisation into responsibilities and its contribution to the
 * M-step sufficient statistics are formed on chip, and only the O(K*D)
 * statistics reach global memory.  The N x K responsibility matrix is never
 * written anywhere (review page, section 2 and section 3; memory O(KD)
 * independent of N).
 *
 * Model (the pages do not print formulas; this is the textbook diagonal GMM):
 *   log p(x) = log sum_k pi_k prod_d Normal(x_d; mu_kd, var_kd)
 *   E-step:  r_nk = pi_k N(x_n | k) / sum_j pi_j N(x_n | j)
 *   M-step:  pi_k = N_k / N,  mu_k = sum_n r_nk x_n / N_k,
 *            var_kd = max(sum_n r_nk (x_nd - mu_kd)^2 / N_k, var_floor)
 *   with N_k = sum_n r_nk.  A component with N_k <= 1e-12 N keeps its mean and
 *   variance and gets pi_k = N_k / N; a component with pi_k = 0 has
 *   responsibility 0 everywhere.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All array pointers are DEVICE pointers owned by the caller unless stated.
 *    The library never allocates or frees device memory and never copies data
 *    between host and device, except where an entry point says so.
 *  - X is N x D, row-major, contiguous, of type problem->xdtype (fp32 or bf16),
 *    16-byte aligned, with D * sizeof(element) a multiple of 16 bytes.
 *  - w is K floats; mu and var are K x D floats, row-major (component-major).
 *    Parameters are in the data's own units.
 *  - ws is a caller-owned device workspace of at least gmm_workspace_size()
 *    bytes, 256-byte aligned.  Its size depends on D, K, the dtype and the
 *    device, never on N.  Calls that share a workspace must be ordered on one
 *    stream.  (gmm_ivf_build, which files points into lists after the fit, has
 *    a workspace of its own, sized by gmm_ivf_workspace_size.)
 *  - stream is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Every entry point only enqueues work on it and returns without
 *    waiting, except gmm_device_status.
 *  - Errors found on the host (null pointers, sizes, alignment, a workspace
 *    that is too small) are returned before anything is enqueued.  Errors found
 *    on the device (a non-finite input, a bounded wait that gave up) are
 *    recorded in a status word inside the workspace; gmm_device_status reads
 *    and clears it.  No entry point aborts, traps or falls back to the CPU.
 */
#ifndef SCEM_GMM_H
#define SCEM_GMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GMM_OK = 0,
  GMM_ERR_INVALID_ARG = 1, /* null pointer, N < 1, D < 1, K < 1, m out of range, ... */
  GMM_ERR_UNSUPPORTED = 2, /* alignment or a shape this build does not handle */
  GMM_ERR_CUDA = 3,        /* a CUDA runtime call failed (no device, launch error, ...) */
  GMM_ERR_NUMERIC = 4,     /* the device saw a NaN/Inf in X or an invalid parameter */
  GMM_ERR_TIMEOUT = 5,     /* a bounded device-side wait gave up */
  GMM_ERR_WORKSPACE = 6    /* workspace null, misaligned or smaller than required */
} gmm_status;

typedef enum { GMM_F32 = 0, GMM_BF16 = 1 } gmm_dtype;

typedef enum {
  GMM_INIT_VAR_ONE = 0, /* every variance starts at 1 */
  GMM_INIT_VAR_DATA = 1 /* every component starts at the per-dimension (biased)
                           sample variance of X, floored */
} gmm_init_var;

typedef struct {
  int64_t N;       /* number of points, >= 1 */
  int32_t D;       /* dimensions, >= 1 */
  int32_t K;       /* mixture components, >= 1 */
  int32_t xdtype;  /* gmm_dtype of X */
  float var_floor; /* variance floor applied by the M-step and the data-variance init, >= 0 */
} gmm_problem;

/* Device status bits recorded in the workspace (see gmm_device_status). */
#define GMM_DEVFLAG_NONFINITE_X 0x1u     /* a NaN or Inf element in X */
#define GMM_DEVFLAG_BAD_PARAMS 0x2u      /* w < 0, var <= 0 or a non-finite parameter */
#define GMM_DEVFLAG_WAIT_TIMEOUT 0x4u    /* a bounded spin on a barrier gave up */
#define GMM_DEVFLAG_X_RANGE 0x8u         /* an element of X lies so far from the mixture mean
                                            (over 240 scale units, about 480 mixture standard
                                            deviations) that the tensor-core path clipped it */
#define GMM_DEVFLAG_BAD_INDEX 0x10u      /* gmm_ivf_build: a component index outside [0, K)
                                            or repeated within one point's row */

/* How the library runs a problem on the current device (see gmm_plan). */
typedef struct {
  int32_t tensor_cores; /* 1: the tcgen05 tensor-core kernel runs the problem; 0: no
                           tensor-core plan (D > 1024, D not a multiple of 4, or no
                           cluster shape fits), and the EM calls return
                           GMM_ERR_UNSUPPORTED */
  int32_t cluster_ctas; /* tensor cores: CTAs per thread-block cluster, 128 components each */
  int32_t groups;       /* tensor cores: component groups.  1: one fused pass, the row
                           normalisation exchanged inside the cluster.  > 1: per chunk of
                           rows, a pass that writes each group's (max, sum-exp) per row
                           to a row buffer, then the statistics pass */
  int32_t fit_one_launch; /* 1: gmm_fit runs all its iterations in one launch of one
                             cluster, X held in the cluster's shared memory (small N * D) */
  int64_t chunk_rows;   /* groups > 1: rows per chunk (fixed by D and K, not by N), else 0 */
} gmm_plan_info;

/* Fills *info for problem p on the current device.  Errors as gmm_workspace_size. */
gmm_status gmm_plan(const gmm_problem* p, gmm_plan_info* info);

/*
 * Bytes of device workspace needed for problem p on the CURRENT device.
 * The value depends on (D, K, xdtype) and the device's SM count only: it is
 * identical for every N (the O(K*D) memory bound of the review page, section 3).
 * Returns GMM_ERR_INVALID_ARG for bad arguments, GMM_ERR_CUDA if no device.
 */
gmm_status gmm_workspace_size(const gmm_problem* p, size_t* bytes);

/*
 * Initial parameters from a seed.  The review page (section 3) gives no
 * initialisation; this one is the library's definition.  mu_k = X[row_k] for
 * K distinct rows drawn uniformly without replacement (requires K <= N),
 * w_k = 1/K, and var = 1 (GMM_INIT_VAR_ONE) or the per-dimension biased sample
 * variance of X, max(., var_floor), for every component (GMM_INIT_VAR_DATA).
 * Writes w, mu, var.
 *
 * The rows are chosen on the host, reproducibly from `seed`: Floyd's sampling
 * algorithm (for j = N-K .. N-1: t uniform in [0, j]; take t, or j if t was
 * taken; row_k is the index taken at step k) drawing its uniform integers from
 * SplitMix64 (Steele, Lea and Flood, OOPSLA 2014) started at state `seed`,
 * output i = mix(seed + (i+1) * 0x9E3779B97F4A7C15); an output x gives
 * x mod n when x < 2^64 - (2^64 mod n) and is redrawn otherwise.  Any other
 * implementation of these two published definitions picks the same rows.
 * Errors: as gmm_em_step, plus GMM_ERR_INVALID_ARG for K > N or a bad
 * init_var.
 */
gmm_status gmm_init(const gmm_problem* p, const void* X, uint64_t seed, int32_t init_var,
                    float* w, float* mu, float* var, void* ws, size_t ws_bytes, void* stream);

/*
 * gmm_init with the K rows chosen by the caller: mu_k = X[rows_host[k]] (HOST
 * array of K int64 in [0, N); repeats allowed), the rest as gmm_init.  The
 * indices are copied to the workspace on `stream`: from pageable memory the
 * copy has read them when the call returns; from pinned (page-locked) memory
 * the array must stay unchanged until the stream has reached this call.
 */
gmm_status gmm_init_rows(const gmm_problem* p, const void* X, const int64_t* rows_host,
                         int32_t init_var, float* w, float* mu, float* var, void* ws,
                         size_t ws_bytes, void* stream);

/*
 * One fused EM iteration, in place: (w, mu, var) <- M-step(E-step(X; w, mu, var)).
 * loglik (device, 1 double, may be NULL) receives LL of the INPUT parameters,
 * sum_n log p(x_n), including the -D/2 log(2 pi) term.
 * The N x K responsibilities exist only on chip (review page, sections 2-3).
 * Runs on the tensor cores; a shape without a tensor-core plan (gmm_plan)
 * returns GMM_ERR_UNSUPPORTED before any launch.
 */
gmm_status gmm_em_step(const gmm_problem* p, const void* X, float* w, float* mu, float* var,
                       double* loglik, void* ws, size_t ws_bytes, void* stream);

/*
 * The two halves of gmm_em_step, for row-sharded EM (each device holds a row
 * shard of X; the statistics of all shards are summed between the halves).
 *
 * gmm_estep_stats: E-step over the rows of X and their sufficient statistics,
 * reduced in a fixed order to fp64, into stats (device, K*(2D+1)+1 doubles):
 *   stats = [ N_k (K) | A (K x D) | B (K x D) | LL ]
 *   N_k = sum_n r_nk, A_kd = sum_n r_nk (x_nd - mu_kd), B_kd = sum_n r_nk (x_nd - mu_kd)^2
 * (moments about the input means, data units), LL = sum_n log p(x_n).
 * Statistics of disjoint row sets add elementwise.  Parameters unchanged.
 *
 * gmm_mstep: M-step, in place (see the model at the top), from the
 * statistics of nshards >= 1 disjoint row shards holding p->N points in
 * total, stored as nshards consecutive buffers (device, nshards x
 * (K*(2D+1)+1) doubles, e.g. the output of an all-gather); they are summed in
 * shard order, so the result does not depend on how the shards were
 * computed.  loglik (device, may be NULL) receives the summed LL.  p->D, p->K
 * and p->var_floor as for the shards; no X and no workspace are used.
 */
gmm_status gmm_estep_stats(const gmm_problem* p, const void* X, const float* w, const float* mu,
                           const float* var, double* stats, void* ws, size_t ws_bytes,
                           void* stream);
gmm_status gmm_mstep(const gmm_problem* p, const double* stats, int32_t nshards, float* w,
                     float* mu, float* var, double* loglik, void* stream);

/*
 * gmm_em_step without a caller-provided workspace, for callers that are not
 * allowed to obtain device memory themselves: for example a plug-in running
 * inside a host application that owns the whole device-memory budget and
 * exposes no allocator, or a latency-bound loop that must not call cudaMalloc
 * because it blocks the whole device.  It performs no device allocation of
 * any kind (no cudaMalloc, no cudaFree, no allocating library routine).
 * The Flash-GMM pages have no counterpart to this entry point.
 *
 * Scratch: a fixed 32 MiB array compiled into this library, present on every
 * device that loads the library until the process exits.  The first call on a
 * device looks up that array's device address (cudaGetSymbolAddress) and
 * caches it with the CUDA context that was current; a later call under
 * another context (one created after cudaDeviceReset, or a non-primary driver
 * context) looks it up again.  Make the first call on each device and context
 * before any stream capture.  When the statistics slots of the regular
 * workspace do not all fit, fewer CTAs (or clusters) run the fused pass, one
 * slot each, which is slower but gives the same result up to summation order.
 * A tensor-core slot holds K*(2D+1)+1 doubles beside the parameter tables.
 * A problem for which not even one fits, or whose plan's row-chunk buffers
 * (several component groups, or D > 128) exceed the scratch, is rejected with
 * GMM_ERR_UNSUPPORTED and a message on stderr.
 *
 * Every call on a device uses the same array and it keeps the previous call's
 * contents; each call resets the status word and rewrites everything else it
 * reads.  Calls whose work overlaps on the GPU (different streams, or several
 * host threads) race on the array and give wrong results: order them on one
 * stream.  dev_flags (device, 1 uint32, may be NULL) receives this call's
 * GMM_DEVFLAG_* bits.  Arguments, loglik and in-place updates are as for
 * gmm_em_step.
 */
gmm_status gmm_em_step_noalloc(const gmm_problem* p, const void* X, float* w, float* mu,
                               float* var, double* loglik, uint32_t* dev_flags, void* stream);

/*
 * Neighbours of the diagonal EM step (the pages present the soft mixture as a
 * replacement for k-means in an IVF coarse quantizer; they print none of
 * these, so each is the textbook form).  All three run the same fused
 * tensor-core E-step and statistics pass as gmm_em_step and take its
 * workspace (gmm_workspace_size).
 *
 * gmm_em_step_hard: classification EM of the diagonal model.  Each point goes
 * wholly to its most probable component (largest log-joint, ties to the lower
 * index); the M-step is gmm_em_step's with those 0/1 responsibilities.
 * labels (device, N int32, may be NULL) receives each point's component;
 * loglik (may be NULL) the classification log-likelihood of the input
 * parameters, sum_n max_k log(pi_k N(x_n | k)).  The decision is made on the
 * tensor-core log-joints: points whose two best components lie within about
 * 1e-3 nats may go to either.  GMM_ERR_UNSUPPORTED for shapes without a
 * tensor-core plan (gmm_plan).
 *
 * gmm_em_step_spherical: soft EM with covariance s2_k * I: s2 is K floats
 * (device, in place); the M-step variance is the mean over dimensions of the
 * per-dimension variance about the new mean, floored at var_floor.  Any
 * shape gmm_em_step takes.
 *
 * gmm_kmeans_step: one Lloyd step.  centers (device, K x D, in place) move to
 * the mean of their points (a centre with no point stays); labels (may be
 * NULL) gets each point's nearest centre (squared Euclidean distance, ties to
 * the lower index, decided like gmm_em_step_hard's); inertia (device, 1
 * double, may be NULL) the sum of squared distances to the input centres.
 * Computed as hard EM with equal weights and one variance shared by every
 * component and dimension.  GMM_ERR_UNSUPPORTED as gmm_em_step_hard.
 */
gmm_status gmm_em_step_hard(const gmm_problem* p, const void* X, float* w, float* mu,
                            float* var, int32_t* labels, double* loglik, void* ws,
                            size_t ws_bytes, void* stream);
gmm_status gmm_em_step_spherical(const gmm_problem* p, const void* X, float* w, float* mu,
                                 float* s2, double* loglik, void* ws, size_t ws_bytes,
                                 void* stream);
gmm_status gmm_kmeans_step(const gmm_problem* p, const void* X, float* centers, int32_t* labels,
                           double* inertia, void* ws, size_t ws_bytes, void* stream);

/*
 * iters EM iterations in place.  ll_history (device, iters doubles, may be
 * NULL) receives LL(theta_t) for t = 0 .. iters-1, each of the parameters that
 * iteration started from.  When the data fit in the shared memory of one
 * thread-block cluster (gmm_plan's fit_one_launch; about N * D <= 8e5 fp32
 * values), all iterations run in a single launch: direct-form E-step on the
 * CUDA cores, statistics in fp64 exchanged over distributed shared memory,
 * the M-step on chip, parameters written back once.  Otherwise each iteration
 * is gmm_em_step.
 */
gmm_status gmm_fit(const gmm_problem* p, const void* X, int32_t iters, float* w, float* mu,
                   float* var, double* ll_history, void* ws, size_t ws_bytes, void* stream);

/*
 * One EM iteration with X in HOST memory: the out-of-core form, for data larger
 * than the device (Flash-GMM abstract: datasets far larger than fit before on one
 * device, since the method's device memory is O(K*D) whatever N is).
 *
 * X_host (N x D row-major, p->xdtype, HOST memory) is copied chunk_rows rows at
 * a time into two device staging buffers on copy_stream, while stream runs the
 * fused E-step and statistics pass on the other buffer.  Each chunk's fp64
 * statistics are added, in chunk order, into one running total, and one
 * M-step follows, so the result is the EM iteration of gmm_em_step on the same
 * rows (the statistics are summed in another order: equal up to rounding, and
 * deterministic for a given chunk_rows).  *loglik gets LL of the input
 * parameters.
 *
 *   X_host       should be pinned (cudaHostAlloc / cudaHostRegister) for the
 *                copies to overlap the E-step; pageable memory works, without
 *                overlap.  It must stay valid and unchanged until stream has
 *                completed the call's work.
 *   chunk_rows   >= 1; rows per copy (the last chunk may hold fewer).
 *   staging      device, 256-byte aligned, gmm_host_staging_size(p, chunk_rows)
 *                bytes: two chunks of X plus two statistics buffers.
 *   ws           the workspace of gmm_workspace_size(p), as for gmm_em_step.
 *   stream, copy_stream  cudaStream_t as void*; they may be the same stream
 *                (no overlap).  The call returns once everything is enqueued.
 * Errors: as gmm_em_step, plus GMM_ERR_INVALID_ARG for chunk_rows < 1 or a null
 * X_host and GMM_ERR_WORKSPACE for missing, misaligned or short staging.
 */
gmm_status gmm_host_staging_size(const gmm_problem* p, int64_t chunk_rows, size_t* bytes);
gmm_status gmm_em_step_host(const gmm_problem* p, const void* X_host, int64_t chunk_rows,
                            void* staging, size_t staging_bytes, float* w, float* mu, float* var,
                            double* loglik, void* ws, size_t ws_bytes, void* stream,
                            void* copy_stream);

/* LL(theta) of the given parameters into *loglik (device, 1 double).  Parameters unchanged. */
gmm_status gmm_loglik(const gmm_problem* p, const void* X, const float* w, const float* mu,
                      const float* var, double* loglik, void* ws, size_t ws_bytes,
                      void* stream);

/*
 * Multi-assignment of each point to its m most responsible components, for
 * placing border vectors in several IVF lists (Flash-GMM abstract: the
 * responsibilities decide which clusters a vector near a cluster border joins).
 * idx (device, N x m int32) gets component indices ordered by responsibility,
 * descending, equal responsibilities in ascending index order; resp (device,
 * N x m float) gets those responsibilities.  1 <= m <= min(K, 8).
 */
gmm_status gmm_assign_topm(const gmm_problem* p, const void* X, const float* w,
                           const float* mu, const float* var, int32_t m, int32_t* idx,
                           float* resp, void* ws, size_t ws_bytes, void* stream);

/*
 * Inverted lists of an IVF coarse quantizer from a top-m assignment: each point
 * is filed under the clusters its responsibilities choose (Flash-GMM abstract:
 * GMM responsibilities put border vectors into several clusters' lists).  The
 * pages give no rule; this library's: point n joins the list of idx[n][0]
 * always, and the list of idx[n][j] (j >= 1) when resp[n][j] >= tau, compared
 * in float32.
 *
 *   idx, resp  device, N x m row-major, as gmm_assign_topm returns them
 *              (1 <= m <= min(K, 8)); resp of rank 1 is not read.
 *   tau        the threshold; not NaN (tau > 1 gives a plain partition by the
 *              rank-1 component, tau <= 0 files every point m times).
 *   offsets    device, K + 1 int64: list k is ids[offsets[k] .. offsets[k+1]),
 *              offsets[K] is the number of entries.
 *   ids        device, ids_capacity int64 point indices, ascending inside each
 *              list; ids_capacity >= N * m (the most entries there can be).
 *   ws         device workspace of gmm_ivf_workspace_size(N, K) bytes, 256-byte
 *              aligned, its first word the status word (zero it once; a call
 *              leaves it unchanged unless it raises a bit).  It grows with N up
 *              to a cap: about 64 MiB of per-chunk counts plus 8 bytes per list.
 *
 * The result does not depend on the launch configuration or on timing.  An
 * entry of idx outside [0, K), or repeating an earlier index of its row, is
 * skipped and raises GMM_DEVFLAG_BAD_INDEX, which gmm_device_status reports as
 * GMM_ERR_INVALID_ARG.  Host errors: GMM_ERR_INVALID_ARG (N < 1, K < 1, m out
 * of range, a null pointer, NaN tau, ids_capacity < N * m),
 * GMM_ERR_UNSUPPORTED (K > 65536 or N > 2^40), GMM_ERR_WORKSPACE.
 */
gmm_status gmm_ivf_workspace_size(int64_t N, int32_t K, size_t* bytes);
gmm_status gmm_ivf_build(int64_t N, int32_t K, int32_t m, const int32_t* idx, const float* resp,
                         float tau, int64_t* offsets, int64_t* ids, int64_t ids_capacity,
                         void* ws, size_t ws_bytes, void* stream);

/*
 * Waits for stream, then reads the device status word of ws into *flags
 * (GMM_DEVFLAG_* bits; may be NULL) and, if clear != 0, resets it to 0.
 * Returns GMM_OK when no bit is set, GMM_ERR_TIMEOUT for the wait bit,
 * GMM_ERR_NUMERIC for the data/parameter/range bits, GMM_ERR_INVALID_ARG for
 * the index bit.  The only entry point that blocks.
 */
gmm_status gmm_device_status(void* ws, size_t ws_bytes, void* stream, uint32_t* flags,
                             int32_t clear);

/*
 * Tracing hook.  While start_event and stop_event (cudaEvent_t handles passed
 * as void*) are non-NULL, every later call that runs the fused E-step pass
 * records start_event on its stream just before that kernel's launch and
 * stop_event just after it, so the kernel's own duration can be read with
 * cudaEventElapsedTime.  Passing NULL, NULL turns it off.  The setting is
 * process-wide; each handle is read and written atomically, but the pair is not
 * swapped as one, so change it while no other host thread is launching.
 */
gmm_status gmm_trace_fused(void* start_event, void* stop_event);

/*
 * Longest time, in nanoseconds, that any device-side wait of the tensor-core
 * pass spins on a barrier for another warp or CTA before it gives up
 * (default 1e9, one second; 0 restores the default).  A wait that gives up
 * sets GMM_DEVFLAG_WAIT_TIMEOUT in the workspace status word; every other wait
 * of the launch then gives up too, the kernel still waits (up to one second)
 * for its own copies and MMAs in flight, releases its shared and tensor memory
 * and returns, and gmm_device_status reports GMM_ERR_TIMEOUT.  The step's
 * outputs are then not meaningful (restore the parameters), but the device
 * context stays usable.  A budget below the time a tile takes (microseconds)
 * makes every step give up: that is how the timeout path is tested.  The
 * setting is process-wide and applies to launches enqueued after the call.
 */
gmm_status gmm_set_wait_budget(uint64_t ns);

/*
 * Number of kernels this library has enqueued in this process so far (all
 * entry points, all devices), into *count.  For tracing and benchmarking.
 */
gmm_status gmm_launch_count(uint64_t* count);

/* Static, human-readable name of a status code. */
const char* gmm_status_string(gmm_status s);

#ifdef __cplusplus
}
#endif

#endif /* SCEM_GMM_H */
