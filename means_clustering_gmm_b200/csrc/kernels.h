// Internal interface between the C-ABI layer (abi.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gmm_b200.h"

namespace gmmb {

// Views into a GMM workspace (all device pointers into the caller's buffer).
struct GmmWs {
    int *err;          // device error word
    float *nhl;        // [K x d]   -1/(2 var)            (CUDA-core path)
    float *ck;         // [K]       per-component constant (both paths)
    float *lse;        // [N]       per-point l_n (two-sweep paths)
    float *partial;    // [P x K x (1+2d)] partial statistics: fp32 (CUDA-core path)
    double *partial64; // the same region read as fp64 (tensor-core path)
    double *ll_part;   // [T] fp64 per-tile log-likelihood partials
    void *tc;          // tensor-core path parameter pieces (see gmm_tc.cu)
    size_t tc_bytes;
};

struct GmmWsLayout {
    size_t off_nhl, off_ck, off_lse, off_partial, off_llpart, off_tc, total;
    int64_t max_partials, max_ll;
    size_t tc_bytes;
};

GmmWsLayout gmm_ws_layout(int64_t N, int d, int K);
GmmWs gmm_ws_bind(void *ws, const GmmWsLayout &L);

// The host-side argument checks of gmm_em_step; GMM_OK or GMM_ERR_INVALID_ARG.
gmm_status gmm_em_step_check(const void *X, gmm_dtype dtype, int64_t N, int d, int K,
                             const float *means, const float *vars, const float *logw,
                             const double *stats, const float *loglik, const double *loglik_total,
                             const void *ws, size_t ws_bytes, uint32_t flags);

// CUDA-core two-sweep path.  Fills w.partial[0..*num_partials) and
// w.ll_part[0..*num_ll).
cudaError_t launch_gmm_simt(const void *X, gmm_dtype dt, int64_t N, int d, int K,
                            const float *means, const float *vars, const float *logw,
                            const GmmWs &w, float *loglik, int *num_partials, int64_t *num_ll,
                            cudaStream_t s);

// Tensor-core path.  Returns cudaErrorNotSupported when the shape has no
// tensor-core kernel (the caller then uses the CUDA-core path).
bool gmm_tc_supported(gmm_dtype dt, int64_t N, int d, int K, uint32_t flags);
int gmm_tc_regime(gmm_dtype dt, int64_t N, int d, int K, uint32_t flags);  // 1 or 2
// Whether the tensor-core path runs the one-CTA fused kernel (K <= 128, or
// sweep 1 of the two-sweep regime) rather than the two-CTA cluster kernel.
bool gmm_tc_runs_fused(gmm_dtype dt, int64_t N, int d, int K, uint32_t flags);
size_t gmm_tc_ws_bytes(int64_t N, int d, int K);
// Points per chunk of a tensor-core step over N points (all of N unless the
// direct-form score block of N points would pass its bound); the override
// (gmm_set_point_chunk) only makes chunks smaller.
int64_t gmm_tc_chunk_points(int64_t N, int d, int K);
void gmm_tc_set_chunk_override(int64_t points);
int64_t gmm_tc_max_partials(int64_t N, int d, int K);
int64_t gmm_tc_max_ll(int64_t N, int d, int K);
// One chunk: X and N are the chunk's rows, w.lse and loglik point at its
// first point, n_ws is the N the workspace was sized for; accumulate marks
// a later chunk of the call.  *num_partials = -1 when the path reduced its
// statistics into `stats` itself (the small-mixture kernel; when
// accumulate, added to what `stats` holds).
cudaError_t launch_gmm_tc(const void *X, gmm_dtype dt, int64_t N, int64_t n_ws, int d, int K,
                          const float *means, const float *vars, const float *logw,
                          const GmmWs &w, float *loglik, uint32_t flags, int *num_partials,
                          int64_t *num_ll, double *stats, bool accumulate, cudaStream_t s);
// Soft assignment (top-R components per point with r >= tau) on the tensor
// cores; cudaErrorNotSupported for shapes without a tensor-core kernel.
cudaError_t launch_gmm_tc_assign(const void *X, gmm_dtype dt, int64_t N, int64_t n_ws, int d,
                                 int K, const float *means, const float *vars, const float *logw,
                                 const GmmWs &w, float *loglik, int R, float tau, int32_t *ids,
                                 float *resp, bool later, cudaStream_t s);
// The same on CUDA cores (any d): direct-form scores, per-point online
// log-sum-exp and top-R.
cudaError_t launch_gmm_simt_assign(const void *X, gmm_dtype dt, int64_t N, int d, int K,
                                   const float *means, const float *vars, const float *logw,
                                   const GmmWs &w, float *loglik, int R, float tau, int32_t *ids,
                                   float *resp, cudaStream_t s);
// After the reduction: add the statistics of the components the tensor-core
// path scored in the direct form (ill-conditioned ones) into `stats`.
cudaError_t launch_gmm_tc_direct_stats(const void *X, gmm_dtype dt, int64_t N, int64_t n_ws,
                                       int d, int K, const GmmWs &w, double *stats,
                                       cudaStream_t s);

// Deterministic fixed-order reductions and the M-step finalise.
// Partials are fp32 (CUDA-core path) or fp64 (tensor-core path); the sum is
// fp64 in a fixed order either way.  accumulate: add into the output (a
// later point chunk of the same step) instead of writing it.
cudaError_t launch_reduce_stats64(const double *partial, int num_partials, int d, int K,
                                  double *stats, bool accumulate, cudaStream_t s);
cudaError_t launch_reduce_stats(const float *partial, int num_partials, int d,
                                int K, double *stats, cudaStream_t s);
cudaError_t launch_reduce_ll(const double *ll_part, int64_t n, double *out, bool accumulate,
                             cudaStream_t s);
// The finalise of B problems in one launch (problem b at b times the sizes).
cudaError_t launch_finalize_batched(const double *stats, int B, int64_t N, int d, int K,
                                    float var_floor, float *means, float *vars, float *logw,
                                    int *err, cudaStream_t s);
// Attributes of one of the library's kernels (the M-step finalise).
cudaError_t gmm_kernel_attributes(cudaFuncAttributes *a);
cudaError_t launch_finalize(const double *stats, int64_t N, int d, int K, float var_floor,
                            float *means, float *vars, float *logw, int *err, cudaStream_t s);

// k-means.
struct KmWsLayout {
    size_t off_mind, off_hist, off_perm, off_segoff, off_inpart, off_cnorm, off_segin, total;
    int nblk;          // sort chunks per problem
    int assign_tiles;  // assignment tiles per problem
};
KmWsLayout km_ws_layout(int B, int64_t N, int d, int K);
// After a kmeans_step (B = 1) on workspace `ws`: per cluster, the variance of
// its members about `means` (the member means), two-pass in fp64, clamped at
// var_floor; an empty cluster gets variance 1.  Reads the step's segments.
cudaError_t launch_km_member_vars(const void *X, gmm_dtype dt, int64_t N, int d, int K,
                                  const void *ws, const float *means, float var_floor,
                                  float *vars, cudaStream_t s);
cudaError_t launch_kmeans(const void *X, gmm_dtype dt, int B, int64_t N, int d, int K,
                          const float *C, int32_t *ids, float *newC, int32_t *counts,
                          double *inertia, void *ws, const KmWsLayout &L, uint32_t flags,
                          cudaStream_t s);

}  // namespace gmmb
