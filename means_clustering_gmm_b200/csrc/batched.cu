// Batched GMM: B independent diagonal mixtures over B point sets of the same
// shape (N x d, K components), the GMM counterpart of the batched Lloyd step
// ("Flash-KMeans gor k-means realtime-venligt pa GPU ...", section
// "FlashAssign gor tildelingen hurtig": batches of independent problems).
//
// Problem b reads X + b N d, its parameters at b K d / b K, writes its
// statistics at b K (1 + 2d), its log-likelihoods at b N and its total at b,
// and owns the b-th slice of the workspace (one gmm_em_step workspace each).
// Every problem runs the fused E-step kernels of gmm_em_step unchanged, in
// problem order on the caller's stream; the M-step finalise of all problems
// is one launch over (component, feature) x problem.  After the problems, one
// kernel folds their device error words into problem 0's (the first recorded
// code of the lowest problem wins), so gmm_last_error(ws) reports the batch.
#include "common.cuh"
#include "kernels.h"

namespace gmmb {
namespace {

size_t batch_stride(int64_t N, int d, int K, gmm_dtype dt) {
    return align_up(gmm_workspace_size(N, d, K, dt));
}

// Problem 0's word keeps the first code of the lowest problem that recorded
// one; the other problems' words are cleared for the next call.
__global__ void fold_errors_kernel(char *ws, size_t stride, int B) {
    int *e0 = (int *)ws;
    int first = *e0;
    for (int b = 1; b < B; ++b) {
        int *eb = (int *)(ws + (size_t)b * stride);
        if (first == 0) first = *eb;
        *eb = 0;
    }
    *e0 = first;
}

__global__ void clear_errors_kernel(char *ws, size_t stride, int B) {
    for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < B; b += gridDim.x * blockDim.x)
        *(int *)(ws + (size_t)b * stride) = 0;
}

bool is_aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

}  // namespace
}  // namespace gmmb

using namespace gmmb;

extern "C" size_t gmm_batched_workspace_size(int B, int64_t N, int d, int K, gmm_dtype dtype) {
    if (B < 1 || gmm_workspace_size(N, d, K, dtype) == 0) return 0;
    return (size_t)B * batch_stride(N, d, K, dtype);
}

extern "C" gmm_status gmm_em_step_batched(const void *X, gmm_dtype dtype, int B, int64_t N, int d,
                                          int K, const float *means, const float *vars,
                                          const float *logw, double *stats, float *loglik,
                                          double *loglik_total, void *ws, size_t ws_bytes,
                                          uint32_t flags, void *stream) {
    const size_t need = gmm_batched_workspace_size(B, N, d, K, dtype);
    if (need == 0 || ws_bytes < need) return GMM_ERR_INVALID_ARG;
    const size_t es = dtype == GMM_F32 ? 4 : 2;
    // every problem's rows must start on a 16-byte boundary
    if (((size_t)N * d * es) % 16 != 0) return GMM_ERR_INVALID_ARG;
    const size_t stride = batch_stride(N, d, K, dtype);
    // host checks of every problem before the first launch
    for (int b = 0; b < B; ++b) {
        const gmm_status chk = gmm_em_step_check(
            (const char *)X + (size_t)b * N * d * es, dtype, N, d, K,
            means + (size_t)b * K * d, vars + (size_t)b * K * d, logw + (size_t)b * K,
            stats + (size_t)b * K * (1 + 2 * (size_t)d), loglik ? loglik + (size_t)b * N : nullptr,
            loglik_total ? loglik_total + b : nullptr, (char *)ws + (size_t)b * stride, stride,
            flags);
        if (chk != GMM_OK) return chk;
        if (!X || !means || !vars || !logw || !stats) return GMM_ERR_INVALID_ARG;
    }
    for (int b = 0; b < B; ++b) {
        const gmm_status st = gmm_em_step(
            (const char *)X + (size_t)b * N * d * es, dtype, N, d, K, means + (size_t)b * K * d,
            vars + (size_t)b * K * d, logw + (size_t)b * K,
            stats + (size_t)b * K * (1 + 2 * (size_t)d), loglik ? loglik + (size_t)b * N : nullptr,
            loglik_total ? loglik_total + b : nullptr, (char *)ws + (size_t)b * stride, stride,
            flags, stream);
        if (st != GMM_OK) return st;
    }
    if (B > 1) {
        fold_errors_kernel<<<1, 1, 0, (cudaStream_t)stream>>>((char *)ws, stride, B);
        note_launches(1);
    }
    return cudaGetLastError() == cudaSuccess ? GMM_OK : GMM_ERR_CUDA;
}

extern "C" gmm_status gmm_finalize_batched(const double *stats, int B, int64_t N, int d, int K,
                                           float var_floor, float *means, float *vars,
                                           float *logw, void *ws, size_t ws_bytes, void *stream) {
    if (B < 1 || N < 1 || d < 1 || d > GMM_MAX_D || K < 1 || K > GMM_MAX_K) return GMM_ERR_INVALID_ARG;
    if (!stats || !means || !vars || !logw || !ws || !(var_floor > 0.f)) return GMM_ERR_INVALID_ARG;
    if (!is_aligned(stats, 8) || !is_aligned(means, 4) || !is_aligned(vars, 4) ||
        !is_aligned(logw, 4) || !is_aligned(ws, kAlign) || ws_bytes < kAlign)
        return GMM_ERR_INVALID_ARG;
    // the error word is problem 0's (the first int of the workspace)
    const cudaError_t e = launch_finalize_batched(stats, B, N, d, K, var_floor, means, vars, logw,
                                                  (int *)ws, (cudaStream_t)stream);
    if (e != cudaSuccess) return GMM_ERR_CUDA;
    note_launches(1);
    return GMM_OK;
}

extern "C" gmm_status gmm_batched_workspace_init(void *ws, int B, int64_t N, int d, int K,
                                                 gmm_dtype dtype, void *stream) {
    const size_t need = gmm_batched_workspace_size(B, N, d, K, dtype);
    if (!ws || need == 0 || !is_aligned(ws, kAlign)) return GMM_ERR_INVALID_ARG;
    clear_errors_kernel<<<(B + 255) / 256, 256, 0, (cudaStream_t)stream>>>(
        (char *)ws, batch_stride(N, d, K, dtype), B);
    note_launches(1);
    return cudaGetLastError() == cudaSuccess ? GMM_OK : GMM_ERR_CUDA;
}
