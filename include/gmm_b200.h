/*
 * gmm_b200.h -- C ABI of the B200 (sm_100a) fused GMM-EM / Lloyd k-means
 * library (libgmm_b200.so).
 *
 * The library implements one data-parallel hot path:
 *   - one expectation-maximisation iteration of a diagonal-covariance Gaussian
 *     mixture over N points x K components x d features that never writes the
 *     N x K score/responsibility matrix to memory: scoring, log-sum-exp
 *     normalisation across K and accumulation of the responsibility-weighted
 *     sufficient statistics happen on chip ("Flash-GMM: a memory-efficient
 *     kernel for scalable soft clustering", abstract; "Turbo-GMM:
 *     FlashAttention-Inspired GPU-Accelerated Gaussian Mixture Model",
 *     abstract), followed by the M-step finalise;
 *   - Lloyd k-means as its hard-assignment special case: a fused distance +
 *     online argmin assignment, then a sort-inverse centroid update (argsort
 *     of the ids, segmented reductions, no per-point atomics)
 *     ("Flash-KMeans gor k-means realtime-venligt pa GPU ...", sections
 *     "FlashAssign gor tildelingen hurtig" and "Centroid-opdatering uden
 *     atomics i stormvejr").
 *
 * Conventions shared by every entry point
 *   - Every pointer argument is a DEVICE pointer owned by the caller unless
 *     stated otherwise.  The library allocates no memory on these paths; the
 *     caller passes a device workspace of at least *_workspace_size() bytes,
 *     256-byte aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and never synchronise, except gmm_last_error().
 *   - Arguments are validated on the host before anything is launched.  A
 *     non-OK status from the call itself means nothing was launched.
 *   - Conditions detected on the device (non-finite parameters after the
 *     M-step, input values outside the range of the tensor-core path, a
 *     bounded wait that ran out) are recorded in an error word inside the
 *     workspace and returned by gmm_last_error().
 *   - Results are deterministic.  Partial statistics are summed in a fixed
 *     order.  The tensor-core kernels move their on-chip statistics into a
 *     per-CTA fp64 partial row with fp64 reductions (red.global.add.f64), but
 *     every element of such a row has exactly one writer thread, whose
 *     operations on it stay in program order, so the sum does not depend on
 *     scheduling.  No two threads ever add into the same element.  Calls that
 *     share a workspace must not overlap in time on the device.
 */
#ifndef GMM_B200_H
#define GMM_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gmm_status {
    GMM_OK = 0,
    GMM_ERR_INVALID_ARG = 1,  /* NULL pointer, size <= 0 or above a limit,
                                 misaligned pointer, workspace too small */
    GMM_ERR_UNSUPPORTED = 2,  /* no kernel for this dtype / shape / flag */
    GMM_ERR_CUDA = 3,         /* a launch or CUDA runtime call failed */
    GMM_ERR_TIMEOUT = 4,      /* device: a bounded wait ran out */
    GMM_ERR_NONFINITE = 5,    /* device: NaN/Inf in the updated parameters */
    GMM_ERR_RANGE = 6         /* device: the tensor-core path cannot
                                 represent the parameters accurately enough
                                 (a component whose pieces fall outside the
                                 fp16 range), or more components with
                                 sum_j mu^2/var above 2^14 than the
                                 direct-form slots (64; K/16 for
                                 1024 < K <= 2048; K/8 above, at most 512);
                                 results are invalid.  Large
                                 data values are not an error: X is scaled
                                 by an exact power of two per call (see
                                 gmm_em_step) */
} gmm_status;

typedef enum gmm_dtype {
    GMM_F32 = 0,   /* IEEE binary32 */
    GMM_BF16 = 1,  /* bfloat16 */
    GMM_F16 = 2    /* IEEE binary16 */
} gmm_dtype;

/* Flags for gmm_em_step / kmeans_step.  They only select between kernels
 * that compute the same result; they exist for testing. */
#define GMM_FLAG_NONE            0u
#define GMM_FLAG_FORCE_TWO_SWEEP 1u  /* GMM: run the two-sweep regime even if
                                        the single sweep fits on chip */
#define GMM_FLAG_FORCE_SIMT      2u  /* run the CUDA-core kernels instead of
                                        the tcgen05 tensor-core kernels */
#define GMM_FLAG_TEST_STALL      4u  /* GMM, testing the failure path only:
                                        one pipeline stage of the first CTA
                                        of the one-CTA tensor-core kernel is
                                        withheld, so its bounded wait runs out
                                        (about 2 s) and the call records
                                        GMM_ERR_TIMEOUT; results are invalid.
                                        GMM_ERR_UNSUPPORTED for shapes that do
                                        not run that kernel (K in 129..256
                                        without FORCE_TWO_SWEEP, or the
                                        CUDA-core path) */

/* Library limits (validated on the host). */
#define GMM_MAX_D 1024
#define GMM_MAX_K 65536
#define KMEANS_MAX_K 4096

/* Human-readable name of a status code (static string). */
const char *gmm_status_string(gmm_status s);

/* Library ABI version: 100 * major + minor. */
int gmm_version(void);

/*
 * Clears the device error word at the start of a freshly allocated workspace
 * (GMM or k-means).  Call once after allocating a workspace and before its
 * first use; asynchronous on `stream`.
 */
gmm_status gmm_workspace_init(void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------ GMM */

/*
 * Which kernels gmm_em_step runs for this problem and flags:
 *   0 = CUDA-core two-sweep kernels,
 *   1 = tcgen05 single sweep (whole component axis on chip),
 *   2 = tcgen05 two sweeps (scores recomputed in the second sweep),
 *  -1 = invalid sizes.
 */
int gmm_regime(int64_t N, int d, int K, gmm_dtype dtype, uint32_t flags);

/*
 * Bytes of device workspace gmm_em_step needs for this problem (large enough
 * for every regime and flag).  Returns 0 for invalid sizes.  Nothing of size
 * N x K is held: beyond fixed-size parts the workspace grows with N by the
 * per-point l_n (4 bytes a point) and the direct-form scores of one point
 * chunk (see gmm_point_chunk), at most 512 MiB.
 */
size_t gmm_workspace_size(int64_t N, int d, int K, gmm_dtype dtype);

/*
 * Points per chunk of gmm_em_step / gmm_soft_assign on this problem: N when
 * the call runs in one piece (always on the CUDA-core kernels), else the
 * size of every chunk but the last, a multiple of 128.  -1 for invalid
 * sizes.  Host-only; no device work.
 */
int64_t gmm_point_chunk(int64_t N, int d, int K, gmm_dtype dtype, uint32_t flags);

/*
 * Tuning and testing: cap the points per chunk of later tensor-core calls
 * at `points` (rounded up to a multiple of 128); 0 restores the automatic
 * size.  It can only make chunks smaller than the workspace allows, so
 * workspaces sized before or after the call stay valid.  Process-wide; not
 * thread-safe.  GMM_ERR_INVALID_ARG for points < 0.
 */
gmm_status gmm_set_point_chunk(int64_t points);

/*
 * One fused E-step of a diagonal-covariance GMM plus the accumulation of the
 * sufficient statistics.
 *
 * Operation (per "Turbo-GMM ...", abstract: score N points against K
 * components, normalise the responsibilities, accumulate sufficient
 * statistics; equivalent to standard EM in real arithmetic):
 *   s_nk  = log w_k - 1/2 sum_j [ log(2 pi var_kj) + (x_nj - mu_kj)^2 / var_kj ]
 *   l_n   = log sum_k exp(s_nk)                 (per-point log-likelihood)
 *   r_nk  = exp(s_nk - l_n)                     (never written to memory)
 *   S0_k  = sum_n r_nk
 *   S1_kj = sum_n r_nk x_nj
 *   S2_kj = sum_n r_nk x_nj^2
 *
 * Arguments
 *   X        [N x d] row-major, element type `dtype`, rows contiguous
 *            (pitch d elements); 16-byte aligned base.  Read only.
 *   N        number of points, 1 <= N < 2^40.
 *   d        features, 1 <= d <= GMM_MAX_D.
 *   K        components, 1 <= K <= GMM_MAX_K.
 *   means    [K x d] fp32 row-major (mu).       Read only.
 *   vars     [K x d] fp32 row-major (var > 0).  Read only.
 *   logw     [K] fp32, natural log of the weights (-inf = empty component).
 *   stats    OUT [K x (1 + 2d)] fp64, laid out S0[K] | S1[K x d] | S2[K x d].
 *   loglik   OUT [N] fp32 per-point l_n, or NULL.
 *   loglik_total OUT [1] fp64, sum_n l_n (fixed-order sum), or NULL.
 *   ws, ws_bytes  device workspace (see gmm_workspace_size).
 *   flags    GMM_FLAG_* (testing only; 0 in normal use).
 *   stream   cudaStream_t.
 * The regime (single sweep with the whole component axis on chip, or two
 * sweeps that recompute the scores) is chosen from the on-chip budget.
 * The tensor-core path first takes max|x| (in the pass over X that also
 * scores the ill-conditioned components in the direct form, or alone when
 * there are none) and feeds the tensor core x 2^-s, with s the exponent that
 * puts max|x| 2^-s in [90.5, 181) (x^2
 * inside the fp16 range, small values as far above fp16's subnormal floor as
 * that allows); the parameters carry 2^s and 2^2s and the statistics are
 * scaled back exactly, so results do not depend on s beyond rounding.  NaN
 * or Inf in X records GMM_ERR_NONFINITE.
 * Point chunks: the tensor-core path runs this whole sequence on one chunk
 * of rows after another (gmm_point_chunk), each with its own max|x| and
 * scale, and adds each chunk's statistics and share of loglik_total (both
 * fp64) to those of the chunks before it, in chunk order.  For a given
 * chunk size the results are reproducible run to run; other chunk sizes
 * change them by fp64 summation order and the per-chunk scale's rounding.
 */
gmm_status gmm_em_step(const void *X, gmm_dtype dtype, int64_t N, int d, int K,
                       const float *means, const float *vars, const float *logw,
                       double *stats, float *loglik, double *loglik_total,
                       void *ws, size_t ws_bytes, uint32_t flags, void *stream);

/*
 * M-step finalise from the statistics of gmm_em_step (textbook maximum
 * likelihood update of a diagonal GMM; the pages print no formula):
 *   N_k = S0_k,  w_k = N_k / N,  mu_kj = S1_kj / N_k,
 *   var_kj = max(S2_kj / N_k - mu_kj^2, var_floor)      (fp64 internally)
 * A component with N_k < 1e-12 * N keeps its previous mean and variance;
 * its log weight becomes log(N_k / N) (-inf when N_k = 0).
 *
 *   stats      [K x (1 + 2d)] fp64 from gmm_em_step.       Read only.
 *   N, d, K    as in gmm_em_step.
 *   var_floor  lower clamp of the variance (> 0).
 *   means, vars [K x d] fp32, logw [K] fp32: IN the parameters that entered
 *              the E-step, OUT the updated parameters (updated in place).
 *   ws, ws_bytes  the workspace of gmm_em_step (holds the error word).
 * A non-finite updated parameter sets GMM_ERR_NONFINITE in the error word.
 */
gmm_status gmm_finalize(const double *stats, int64_t N, int d, int K, float var_floor,
                        float *means, float *vars, float *logw,
                        void *ws, size_t ws_bytes, void *stream);

/*
 * Soft multi-assignment: for every point, the r components with the largest
 * responsibilities r_nk = exp(s_nk - l_n) (in decreasing order; ties to the
 * lower component index), keeping those with r_nk >= tau.  This is the
 * border-vector assignment of a soft coarse quantizer: a point near the
 * border of two clusters is listed in both ("Flash-GMM: a memory-efficient
 * kernel for scalable soft clustering", abstract: soft assignment in the
 * coarse quantizer of an inverted-file index).  The selection runs on chip
 * in the same pass that forms l_n (the scores never reach memory); no
 * statistics are accumulated.
 *
 *   X, dtype, N, d, K, means, vars, logw  as for gmm_em_step.
 *   r          1 <= r <= 8 components kept per point.
 *   tau        0 <= tau <= 1: entries with r_nk < tau are dropped.
 *   ids        OUT [N x r] int32 component indices, -1 past the cut.
 *   resp       OUT [N x r] fp32 responsibilities, 0 past the cut.
 *   loglik     OUT [N] fp32 l_n, or NULL.
 *   ws, ws_bytes  a gmm_em_step workspace (gmm_workspace_size()).
 *   flags      0, or GMM_FLAG_FORCE_SIMT (CUDA-core kernel).
 * Errors as gmm_em_step (GMM_ERR_INVALID_ARG also for r or tau out of range).
 */
gmm_status gmm_soft_assign(const void *X, gmm_dtype dtype, int64_t N, int d, int K,
                           const float *means, const float *vars, const float *logw,
                           int r, float tau, int32_t *ids, float *resp, float *loglik,
                           void *ws, size_t ws_bytes, uint32_t flags, void *stream);

/* ----------------------------------------------------------- batched GMM */

/*
 * B independent mixtures over B point sets of one shape (the batched
 * workloads of "Flash-KMeans gor k-means realtime-venligt pa GPU ...",
 * section "FlashAssign gor tildelingen hurtig", here for the GMM step).
 * Problem b's tensors sit at b times the per-problem sizes:
 *   X [B x N x d], means / vars [B x K x d], logw [B x K],
 *   stats [B x K x (1 + 2d)], loglik [B x N] (or NULL), loglik_total [B]
 *   (or NULL).
 * Each problem is one gmm_em_step (same kernels, same results as B separate
 * calls) on its own slice of the workspace; N * d * sizeof(dtype) must be a
 * multiple of 16 bytes (16-byte aligned rows for every problem).
 */
size_t gmm_batched_workspace_size(int B, int64_t N, int d, int K, gmm_dtype dtype);

/* Clears the device error words of a freshly allocated batched workspace
 * (one per problem).  Call once before its first use; asynchronous. */
gmm_status gmm_batched_workspace_init(void *ws, int B, int64_t N, int d, int K, gmm_dtype dtype,
                                      void *stream);

/*
 * gmm_em_step for every problem.  All problems are checked on the host before
 * the first launch (GMM_ERR_INVALID_ARG / GMM_ERR_UNSUPPORTED as gmm_em_step).
 * A device condition of any problem is reported by gmm_last_error(ws): the
 * first code recorded by the lowest-numbered problem.
 */
gmm_status gmm_em_step_batched(const void *X, gmm_dtype dtype, int B, int64_t N, int d, int K,
                               const float *means, const float *vars, const float *logw,
                               double *stats, float *loglik, double *loglik_total,
                               void *ws, size_t ws_bytes, uint32_t flags, void *stream);

/* gmm_finalize for every problem, in one launch (same arithmetic). */
gmm_status gmm_finalize_batched(const double *stats, int B, int64_t N, int d, int K,
                                float var_floor, float *means, float *vars, float *logw,
                                void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------- EM fit */

/*
 * Bytes of device workspace gmm_fit needs: gmm_workspace_size(N, d, K, dtype)
 * plus the fit's own block (the [K x (1 + 2d)] fp64 statistics and the loop
 * state).  Returns 0 for invalid sizes.
 */
size_t gmm_fit_workspace_size(int64_t N, int d, int K, gmm_dtype dtype);

/*
 * EM iterations until convergence, with the loop and the convergence test on
 * the device.  A soft clustering fitted this way is the pages' drop-in
 * replacement for k-means ("Flash-GMM: a memory-efficient kernel for scalable
 * soft clustering", abstract); each iteration is gmm_em_step followed by
 * gmm_finalize, unchanged.  Iteration t computes L_t = sum_n l_n at the
 * parameters entering it; the loop stops after the iteration in which
 *   |L_t - L_{t-1}| <= tol * |L_t|        (t >= 1; converged)
 * or after max_iters iterations, or when a device condition is recorded in
 * the error word or L_t is not finite.  The parameters then hold the result
 * of that iteration's M-step.
 *
 * The loop is one CUDA graph with a conditional WHILE node (one EM iteration
 * and a one-thread control kernel per pass); it is built on each call,
 * launched on `stream`, and released when it completes.  The host does not
 * wait: read fit_info / loglik_trace after synchronising the stream.
 *
 *   X, dtype, N, d, K, flags  as for gmm_em_step.
 *   means, vars, logw  IN the initial parameters, OUT the fitted ones
 *              (updated in place, [K x d], [K x d], [K] fp32).
 *   max_iters  >= 1.  tol >= 0 (relative).  var_floor > 0 (gmm_finalize).
 *   loglik_trace  OUT [max_iters] fp64 (device), L_t of every iteration run,
 *              or NULL.
 *   fit_info   OUT [2] int (device): iterations run, and 1 if the tolerance
 *              test stopped the loop (0 otherwise), or NULL.
 *   ws, ws_bytes  at least gmm_fit_workspace_size(); its first
 *              gmm_workspace_size() bytes are the EM step's workspace
 *              (gmm_last_error(ws) reads its error word).
 * Errors: GMM_ERR_INVALID_ARG as gmm_em_step, or for max_iters < 1, tol < 0,
 * var_floor <= 0, a misaligned trace or info pointer (nothing launched);
 * GMM_ERR_CUDA if the graph cannot be built or launched (nothing launched).
 * While this call builds its graph, the kernel timer (gmm_set_kernel_timer)
 * is suspended: a conditional graph body cannot record events.
 */
gmm_status gmm_fit(const void *X, gmm_dtype dtype, int64_t N, int d, int K,
                   float *means, float *vars, float *logw, int max_iters, double tol,
                   float var_floor, double *loglik_trace, int *fit_info,
                   void *ws, size_t ws_bytes, uint32_t flags, void *stream);

/* Bytes of device workspace gmm_init_kmeans needs (0 for invalid sizes). */
size_t gmm_init_kmeans_workspace_size(int64_t N, int d, int K);

/*
 * Initial GMM parameters from k-means: `iters` Lloyd iterations (kmeans_step
 * with B = 1) from the centroids in `means`, then the maximum-likelihood
 * M-step of the final hard partition (responsibility 1 for a point's
 * cluster, 0 otherwise):
 *   mu_k  = mean of the members (the last Lloyd update),
 *   var_kj = (1/n_k) sum_members (x_j - mu_kj)^2, clamped at var_floor,
 *   w_k   = max(n_k, 1) / (N + e), e = number of empty clusters,
 * so an empty cluster stays a live component (its centroid as mean, variance
 * 1, one point's weight).  The pages fit GMMs where k-means was used before
 * ("Flash-GMM ...", abstract); this is the usual k-means start of such a fit.
 *
 *   X, dtype, N, d, K  as for kmeans_step with B = 1 (K <= KMEANS_MAX_K).
 *   iters      >= 1 Lloyd iterations.
 *   var_floor  > 0.
 *   means      IN initial centroids [K x d] fp32; OUT the GMM means.
 *   vars, logw OUT [K x d] fp32 and [K] fp32 (natural log).
 *   ids        OUT [N] int32 cluster of each point in the final partition
 *              (the assignment of the last Lloyd iteration), or NULL.
 *   ws, ws_bytes  at least gmm_init_kmeans_workspace_size(); 256-byte aligned.
 */
gmm_status gmm_init_kmeans(const void *X, gmm_dtype dtype, int64_t N, int d, int K, int iters,
                           float var_floor, float *means, float *vars, float *logw,
                           int32_t *ids, void *ws, size_t ws_bytes, void *stream);

/* --------------------------------------------------------------- k-means */

/* Bytes of device workspace kmeans_step needs.  Returns 0 for invalid sizes. */
size_t kmeans_workspace_size(int B, int64_t N, int d, int K);

/*
 * One Lloyd iteration for B independent problems of N points each.
 *   assignment: ids_bn = argmin_k ||x_bn - c_bk||^2 (lowest k on ties),
 *               computed as argmin_k (||c_bk||^2 - 2 x_bn . c_bk) with an
 *               online argmin over centroid tiles (no N x K matrix);
 *   update:     a stable argsort of the ids gives contiguous segments; each
 *               segment's rows are summed in point order; new centroid =
 *               sum / count; an empty cluster keeps its centroid.
 *
 *   X          [B x N x d] row-major, element type `dtype`; 16-byte aligned.
 *   B, N, d, K 1 <= B, 1 <= N < 2^31 / B, 1 <= d <= GMM_MAX_D,
 *              1 <= K <= KMEANS_MAX_K.
 *   centroids  [B x K x d] fp32.                           Read only.
 *   ids        OUT [B x N] int32.
 *   new_centroids OUT [B x K x d] fp32 (may not alias centroids).
 *   counts     OUT [B x K] int32 members per cluster, or NULL.
 *   inertia    OUT [B] fp64 sum of the squared distances to the assigned
 *              centroid (fixed-order sum), or NULL.
 *   ws, ws_bytes, flags, stream  as for gmm_em_step.
 */
gmm_status kmeans_step(const void *X, gmm_dtype dtype, int B, int64_t N, int d, int K,
                       const float *centroids, int32_t *ids, float *new_centroids,
                       int32_t *counts, double *inertia,
                       void *ws, size_t ws_bytes, uint32_t flags, void *stream);

/* ---------------------------------------------------------------- errors */

/*
 * Waits for `stream`, then returns and clears the device-side error word held
 * in the workspace `ws` (GMM_OK if no device condition was recorded), or
 * GMM_ERR_CUDA if a CUDA error is pending on the stream.
 */
gmm_status gmm_last_error(void *ws, void *stream);

/* ------------------------------------------------- no-allocation variant */

/*
 * Size of the library's static device scratch (a file-scope __device__ array,
 * one per device, created when the module loads): the largest workspace
 * gmm_em_step_static can serve.
 */
#define GMM_STATIC_SCRATCH_BYTES ((size_t)32 << 20)

/*
 * gmm_em_step for callers that cannot allocate device memory and hold no
 * workspace: a plain C caller that owns only the input and output buffers
 * and must keep a fixed device-memory footprint (cudaMalloc / cudaFree on its
 * path could fail under memory pressure and synchronise the device).  The
 * pages have no counterpart: their kernels take their scratch from the
 * framework's allocator.
 *
 * Same operation, arguments and results as gmm_em_step, except:
 *   - the workspace is the library's static scratch of
 *     GMM_STATIC_SCRATCH_BYTES; nothing is allocated (no cudaMalloc,
 *     cudaFree or other allocating call, on any call);
 *   - device_status  OUT [1] int (device memory), or NULL: receives the
 *     device-side error word of this call (GMM_OK or a gmm_status), written
 *     on `stream` at the end of the call; the word is cleared at the start
 *     of every call, so each call reports only its own conditions.
 * Returns GMM_ERR_UNSUPPORTED, before any device work, when
 * gmm_workspace_size(N, d, K, dtype) exceeds GMM_STATIC_SCRATCH_BYTES;
 * GMM_ERR_INVALID_ARG as gmm_em_step does, also before any device work (the
 * scratch is not touched); GMM_ERR_CUDA if the scratch's address cannot be
 * obtained or a launch fails.  device_status is written only when the call
 * returns GMM_OK.
 * Set-up: the first call on a device (the current device) looks up the
 * scratch's address with cudaGetSymbolAddress and caches it; make that
 * first call before any stream capture.
 * Concurrency: all calls on a device share one scratch, so calls whose
 * device work overlaps in time (other streams, other host threads) race and
 * corrupt each other's results; serialise them.
 */
gmm_status gmm_em_step_static(const void *X, gmm_dtype dtype, int64_t N, int d, int K,
                              const float *means, const float *vars, const float *logw,
                              double *stats, float *loglik, double *loglik_total,
                              int *device_status, uint32_t flags, void *stream);

/* --------------------------------------------------------------- tracing */

/*
 * Kernel timer: when both are non-NULL, every later gmm_em_step / kmeans_step
 * records `start_event` on its stream right before its dominant kernel (the
 * fused E-step kernel(s), or the k-means assignment) and `stop_event` right
 * after it.  Both are cudaEvent_t handles owned by the caller; pass NULL,
 * NULL to stop.  Process-wide setting; not thread-safe.
 */
gmm_status gmm_set_kernel_timer(void *start_event, void *stop_event);

/*
 * Collecting kernel timer, for calls whose dominant kernel runs more than
 * once (one region per point chunk of gmm_em_step).  After
 * gmm_kernel_timer_begin every region the library would bracket for
 * gmm_set_kernel_timer is bracketed instead by a pair of the library's own
 * events on the launching stream (the caller's pair is then not recorded).
 * gmm_kernel_timer_end stops collecting, waits for those events, writes the
 * first `cap` region durations in milliseconds, in launch order, to `ms`
 * (host memory; may be NULL when cap = 0) and their number to *regions
 * (may be NULL).  GMM_ERR_INVALID_ARG without a begin or for cap < 0 (or
 * cap > 0 with NULL ms); GMM_ERR_CUDA if an event could not be created or
 * read.  Process-wide; not thread-safe; suspended while gmm_fit builds its
 * graph.
 */
gmm_status gmm_kernel_timer_begin(void);
gmm_status gmm_kernel_timer_end(double *ms, int64_t cap, int64_t *regions);

/* Number of kernels this library has launched in this process so far. */
uint64_t gmm_kernel_launch_count(void);

/*
 * Architecture of the device code the library runs on the current device:
 * the binaryVersion that cudaFuncGetAttributes reports for one of its kernels
 * (100 for sm_100a), or -1 if the query fails (no device, or no image for
 * this device).  Diagnostic only; no device work.
 */
int gmm_device_binary_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GMM_B200_H */
