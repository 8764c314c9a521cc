// C ABI of libgmm_b200 (declared in include/gmm_b200.h): host-side argument
// validation, workspace layout and kernel dispatch.  Every step of the
// computation runs in the kernels of this library; there is no host fallback.
#include "common.cuh"
#include "kernels.h"

#include <atomic>
#include <string.h>
#include <vector>

using namespace gmmb;

namespace gmmb {

static std::atomic<uint64_t> g_launches{0};
static cudaEvent_t g_timer_start = nullptr, g_timer_stop = nullptr;
// The collecting timer: event pairs of the library's own ([2i] start,
// [2i + 1] stop), created as needed and kept for reuse; g_pairs_used of them
// hold regions since gmm_kernel_timer_begin.
static bool g_collect = false, g_timer_off = false, g_collect_failed = false;
static std::vector<cudaEvent_t> g_pool;
static size_t g_pairs_used = 0;

void note_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
void timer_begin(cudaStream_t s) {
    if (g_timer_off) return;
    if (g_collect) {
        if (2 * g_pairs_used + 2 > g_pool.size()) {
            cudaEvent_t a = nullptr, b = nullptr;
            if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) {
                if (a) cudaEventDestroy(a);
                (void)cudaGetLastError();
                g_collect_failed = true;
                return;
            }
            g_pool.push_back(a);
            g_pool.push_back(b);
        }
        cudaEventRecord(g_pool[2 * g_pairs_used], s);
        return;
    }
    if (g_timer_start && g_timer_stop) cudaEventRecord(g_timer_start, s);
}
void timer_end(cudaStream_t s) {
    if (g_timer_off) return;
    if (g_collect) {
        if (2 * g_pairs_used + 2 <= g_pool.size()) {
            cudaEventRecord(g_pool[2 * g_pairs_used + 1], s);
            ++g_pairs_used;
        }
        return;
    }
    if (g_timer_start && g_timer_stop) cudaEventRecord(g_timer_stop, s);
}
bool timer_suspend(bool suspend) {
    const bool was = g_timer_off;
    g_timer_off = suspend;
    return was;
}

GmmWsLayout gmm_ws_layout(int64_t N, int d, int K) {
    GmmWsLayout L;
    GmmSimtPlan p = gmm_simt_plan(N, d, K);
    // the partial region holds either path's rows: fp32 for the CUDA-core
    // kernels, fp64 (at most one per 128-point tile) for the tensor-core ones
    const int64_t tcp = gmm_tc_max_partials(N, d, K);
    L.max_partials = p.ranges > tcp ? p.ranges : tcp;
    const size_t part_rows_bytes = (size_t)p.ranges * sizeof(float) > (size_t)tcp * sizeof(double)
                                       ? (size_t)p.ranges * sizeof(float)
                                       : (size_t)tcp * sizeof(double);
    L.max_ll = p.lse_tiles;
    int64_t tcl = gmm_tc_max_ll(N, d, K);
    if (tcl > L.max_ll) L.max_ll = tcl;
    L.tc_bytes = gmm_tc_ws_bytes(N, d, K);
    size_t o = kAlign;  // error word
    L.off_nhl = o;     o = align_up(o + sizeof(float) * (size_t)K * d);
    L.off_ck = o;      o = align_up(o + sizeof(float) * (size_t)K);
    L.off_lse = o;     o = align_up(o + sizeof(float) * (size_t)N);
    L.off_partial = o; o = align_up(o + part_rows_bytes * K * (1 + 2 * (size_t)d));
    L.off_llpart = o;  o = align_up(o + sizeof(double) * (size_t)L.max_ll);
    L.off_tc = o;      o = align_up(o + L.tc_bytes);
    L.total = o;
    return L;
}

GmmWs gmm_ws_bind(void *ws, const GmmWsLayout &L) {
    char *b = (char *)ws;
    GmmWs w;
    w.err = (int *)b;
    w.nhl = (float *)(b + L.off_nhl);
    w.ck = (float *)(b + L.off_ck);
    w.lse = (float *)(b + L.off_lse);
    w.partial = (float *)(b + L.off_partial);
    w.partial64 = (double *)(b + L.off_partial);
    w.ll_part = (double *)(b + L.off_llpart);
    w.tc = b + L.off_tc;
    w.tc_bytes = L.tc_bytes;
    return w;
}

}  // namespace gmmb

static bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

static bool valid_gmm_sizes(int64_t N, int d, int K) {
    return N >= 1 && N < ((int64_t)1 << 40) && d >= 1 && d <= GMM_MAX_D && K >= 1 &&
           K <= GMM_MAX_K;
}

static bool valid_dtype(gmm_dtype dt) { return dt == GMM_F32 || dt == GMM_BF16 || dt == GMM_F16; }

// Every host-side check of gmm_em_step (sizes, dtype, NULL and alignment,
// flags, workspace size), in one place so that callers that wrap the step
// (gmm_em_step_static) can run them before touching any device memory.
gmm_status gmmb::gmm_em_step_check(const void *X, gmm_dtype dtype, int64_t N, int d, int K,
                                   const float *means, const float *vars, const float *logw,
                                   const double *stats, const float *loglik,
                                   const double *loglik_total, const void *ws, size_t ws_bytes,
                                   uint32_t flags) {
    if (!valid_gmm_sizes(N, d, K) || !valid_dtype(dtype)) return GMM_ERR_INVALID_ARG;
    if (!X || !means || !vars || !logw || !stats || !ws) return GMM_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(ws, kAlign) || !aligned(means, 4) || !aligned(vars, 4) ||
        !aligned(logw, 4) || !aligned(stats, 8) || (loglik && !aligned(loglik, 4)) ||
        (loglik_total && !aligned(loglik_total, 8)))
        return GMM_ERR_INVALID_ARG;
    if (flags & ~(GMM_FLAG_FORCE_TWO_SWEEP | GMM_FLAG_FORCE_SIMT | GMM_FLAG_TEST_STALL))
        return GMM_ERR_INVALID_ARG;
    if (ws_bytes < gmm_ws_layout(N, d, K).total) return GMM_ERR_INVALID_ARG;
    if ((flags & GMM_FLAG_TEST_STALL) &&
        ((flags & GMM_FLAG_FORCE_SIMT) || !gmm_tc_supported(dtype, N, d, K, flags) ||
         !gmm_tc_runs_fused(dtype, N, d, K, flags)))
        return GMM_ERR_UNSUPPORTED;
    return GMM_OK;
}

extern "C" {

const char *gmm_status_string(gmm_status s) {
    switch (s) {
        case GMM_OK: return "GMM_OK";
        case GMM_ERR_INVALID_ARG: return "GMM_ERR_INVALID_ARG";
        case GMM_ERR_UNSUPPORTED: return "GMM_ERR_UNSUPPORTED";
        case GMM_ERR_CUDA: return "GMM_ERR_CUDA";
        case GMM_ERR_TIMEOUT: return "GMM_ERR_TIMEOUT";
        case GMM_ERR_NONFINITE: return "GMM_ERR_NONFINITE";
        case GMM_ERR_RANGE: return "GMM_ERR_RANGE";
    }
    return "GMM_ERR_UNKNOWN";
}

int gmm_version(void) { return 100; }

gmm_status gmm_workspace_init(void *ws, size_t ws_bytes, void *stream) {
    if (!ws || !aligned(ws, kAlign) || ws_bytes < kAlign) return GMM_ERR_INVALID_ARG;
    return cudaMemsetAsync(ws, 0, kAlign, (cudaStream_t)stream) == cudaSuccess ? GMM_OK
                                                                                : GMM_ERR_CUDA;
}

int gmm_regime(int64_t N, int d, int K, gmm_dtype dtype, uint32_t flags) {
    if (!valid_gmm_sizes(N, d, K) || !valid_dtype(dtype)) return -1;
    if ((flags & GMM_FLAG_FORCE_SIMT) || !gmm_tc_supported(dtype, N, d, K, flags)) return 0;
    return gmm_tc_regime(dtype, N, d, K, flags);
}

size_t gmm_workspace_size(int64_t N, int d, int K, gmm_dtype dtype) {
    if (!valid_gmm_sizes(N, d, K) || !valid_dtype(dtype)) return 0;
    return gmm_ws_layout(N, d, K).total;
}

gmm_status gmm_em_step(const void *X, gmm_dtype dtype, int64_t N, int d, int K,
                       const float *means, const float *vars, const float *logw,
                       double *stats, float *loglik, double *loglik_total, void *ws,
                       size_t ws_bytes, uint32_t flags, void *stream) {
    const gmm_status chk = gmm_em_step_check(X, dtype, N, d, K, means, vars, logw, stats, loglik,
                                             loglik_total, ws, ws_bytes, flags);
    if (chk != GMM_OK) return chk;
    GmmWsLayout L = gmm_ws_layout(N, d, K);
    GmmWs w = gmm_ws_bind(ws, L);
    cudaStream_t s = (cudaStream_t)stream;
    int nparts = 0;
    int64_t nll = 0;
    cudaError_t e;
    if ((flags & GMM_FLAG_FORCE_SIMT) || !gmm_tc_supported(dtype, N, d, K, flags)) {
        e = launch_gmm_simt(X, dtype, N, d, K, means, vars, logw, w, loglik, &nparts, &nll, s);
        if (e != cudaSuccess) return GMM_ERR_CUDA;
        e = launch_reduce_stats(w.partial, nparts, d, K, stats, s);
        if (e != cudaSuccess) return GMM_ERR_CUDA;
        note_launches(1);
        if (loglik_total) {
            e = launch_reduce_ll(w.ll_part, nll, loglik_total, false, s);
            if (e != cudaSuccess) return GMM_ERR_CUDA;
            note_launches(1);
        }
        return GMM_OK;
    }
    // tensor-core path, chunk by chunk over the points: each chunk runs the
    // whole launch sequence on its rows and adds its statistics and its part
    // of the total log-likelihood to those of the chunks before it, in chunk
    // order
    const int64_t chunk = gmm_tc_chunk_points(N, d, K);
    const size_t row_bytes = (size_t)d * (dtype == GMM_F32 ? 4 : 2);
    for (int64_t n0 = 0; n0 < N; n0 += chunk) {
        const int64_t nc = N - n0 < chunk ? N - n0 : chunk;
        const bool acc = n0 > 0;
        const void *Xc = (const char *)X + (size_t)n0 * row_bytes;
        GmmWs wc = w;
        wc.lse = w.lse + n0;
        e = launch_gmm_tc(Xc, dtype, nc, N, d, K, means, vars, logw, wc, loglik ? loglik + n0 : nullptr,
                          flags, &nparts, &nll, stats, acc, s);
        if (e != cudaSuccess) return GMM_ERR_CUDA;
        if (nparts >= 0) {   // (-1: the kernel path reduced into stats itself)
            e = launch_reduce_stats64(wc.partial64, nparts, d, K, stats, acc, s);
            if (e != cudaSuccess) return GMM_ERR_CUDA;
            note_launches(1);
        }
        // the components the chunk scored in the direct form
        e = launch_gmm_tc_direct_stats(Xc, dtype, nc, N, d, K, wc, stats, s);
        if (e != cudaSuccess) return GMM_ERR_CUDA;
        if (loglik_total) {
            e = launch_reduce_ll(wc.ll_part, nll, loglik_total, acc, s);
            if (e != cudaSuccess) return GMM_ERR_CUDA;
            note_launches(1);
        }
    }
    return GMM_OK;
}

gmm_status gmm_soft_assign(const void *X, gmm_dtype dtype, int64_t N, int d, int K,
                           const float *means, const float *vars, const float *logw, int r,
                           float tau, int32_t *ids, float *resp, float *loglik, void *ws,
                           size_t ws_bytes, uint32_t flags, void *stream) {
    if (!valid_gmm_sizes(N, d, K) || !valid_dtype(dtype)) return GMM_ERR_INVALID_ARG;
    if (r < 1 || r > kTopMax || !(tau >= 0.f && tau <= 1.f)) return GMM_ERR_INVALID_ARG;
    if (!X || !means || !vars || !logw || !ids || !resp || !ws) return GMM_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(ws, kAlign) || !aligned(means, 4) || !aligned(vars, 4) ||
        !aligned(logw, 4) || !aligned(ids, 4) || !aligned(resp, 4) ||
        (loglik && !aligned(loglik, 4)))
        return GMM_ERR_INVALID_ARG;
    if (flags & ~GMM_FLAG_FORCE_SIMT) return GMM_ERR_INVALID_ARG;
    const GmmWsLayout L = gmm_ws_layout(N, d, K);
    if (ws_bytes < L.total) return GMM_ERR_INVALID_ARG;
    const GmmWs w = gmm_ws_bind(ws, L);
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if ((flags & GMM_FLAG_FORCE_SIMT) || !gmm_tc_supported(dtype, N, d, K, flags)) {
        e = launch_gmm_simt_assign(X, dtype, N, d, K, means, vars, logw, w, loglik, r, tau, ids,
                                   resp, s);
        return e == cudaSuccess ? GMM_OK : GMM_ERR_CUDA;
    }
    // tensor-core path, chunk by chunk over the points (as gmm_em_step)
    const int64_t chunk = gmm_tc_chunk_points(N, d, K);
    const size_t row_bytes = (size_t)d * (dtype == GMM_F32 ? 4 : 2);
    for (int64_t n0 = 0; n0 < N; n0 += chunk) {
        const int64_t nc = N - n0 < chunk ? N - n0 : chunk;
        GmmWs wc = w;
        wc.lse = w.lse + n0;
        e = launch_gmm_tc_assign((const char *)X + (size_t)n0 * row_bytes, dtype, nc, N, d, K,
                                 means, vars, logw, wc, loglik ? loglik + n0 : nullptr, r, tau,
                                 ids + (size_t)n0 * r, resp + (size_t)n0 * r, n0 > 0, s);
        if (e != cudaSuccess) return GMM_ERR_CUDA;
    }
    return GMM_OK;
}

gmm_status gmm_finalize(const double *stats, int64_t N, int d, int K, float var_floor,
                        float *means, float *vars, float *logw, void *ws, size_t ws_bytes,
                        void *stream) {
    if (!valid_gmm_sizes(N, d, K)) return GMM_ERR_INVALID_ARG;
    if (!stats || !means || !vars || !logw || !ws) return GMM_ERR_INVALID_ARG;
    if (!(var_floor > 0.f)) return GMM_ERR_INVALID_ARG;
    if (!aligned(stats, 8) || !aligned(means, 4) || !aligned(vars, 4) || !aligned(logw, 4) ||
        !aligned(ws, kAlign) || ws_bytes < kAlign)
        return GMM_ERR_INVALID_ARG;
    cudaError_t e = launch_finalize(stats, N, d, K, var_floor, means, vars, logw, (int *)ws,
                                    (cudaStream_t)stream);
    if (e != cudaSuccess) return GMM_ERR_CUDA;
    note_launches(1);
    return GMM_OK;
}

size_t kmeans_workspace_size(int B, int64_t N, int d, int K) {
    if (B < 1 || N < 1 || d < 1 || d > GMM_MAX_D || K < 1 || K > KMEANS_MAX_K) return 0;
    if ((int64_t)B * N >= ((int64_t)1 << 31)) return 0;
    return km_ws_layout(B, N, d, K).total;
}

gmm_status kmeans_step(const void *X, gmm_dtype dtype, int B, int64_t N, int d, int K,
                       const float *centroids, int32_t *ids, float *new_centroids,
                       int32_t *counts, double *inertia, void *ws, size_t ws_bytes,
                       uint32_t flags, void *stream) {
    if (B < 1 || N < 1 || d < 1 || d > GMM_MAX_D || K < 1 || K > KMEANS_MAX_K ||
        !valid_dtype(dtype))
        return GMM_ERR_INVALID_ARG;
    if ((int64_t)B * N >= ((int64_t)1 << 31)) return GMM_ERR_INVALID_ARG;
    if (!X || !centroids || !ids || !new_centroids || !ws) return GMM_ERR_INVALID_ARG;
    if ((const void *)centroids == (const void *)new_centroids) return GMM_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(ws, kAlign) || !aligned(centroids, 4) || !aligned(ids, 4) ||
        !aligned(new_centroids, 4) || (counts && !aligned(counts, 4)) ||
        (inertia && !aligned(inertia, 8)))
        return GMM_ERR_INVALID_ARG;
    if (flags & ~(GMM_FLAG_FORCE_SIMT)) return GMM_ERR_INVALID_ARG;
    KmWsLayout L = km_ws_layout(B, N, d, K);
    if (ws_bytes < L.total) return GMM_ERR_INVALID_ARG;
    cudaError_t e = launch_kmeans(X, dtype, B, N, d, K, centroids, ids, new_centroids, counts,
                                  inertia, ws, L, flags, (cudaStream_t)stream);
    return e == cudaSuccess ? GMM_OK : GMM_ERR_CUDA;
}

gmm_status gmm_last_error(void *ws, void *stream) {
    if (!ws) return GMM_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GMM_ERR_CUDA;
    int code = 0;
    if (cudaMemcpy(&code, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return GMM_ERR_CUDA;
    if (code != 0 && cudaMemset(ws, 0, sizeof(int)) != cudaSuccess) return GMM_ERR_CUDA;
    return (gmm_status)code;
}

gmm_status gmm_set_kernel_timer(void *start_event, void *stop_event) {
    if ((start_event == nullptr) != (stop_event == nullptr)) return GMM_ERR_INVALID_ARG;
    g_timer_start = (cudaEvent_t)start_event;
    g_timer_stop = (cudaEvent_t)stop_event;
    return GMM_OK;
}

gmm_status gmm_kernel_timer_begin(void) {
    g_collect = true;
    g_collect_failed = false;
    g_pairs_used = 0;
    return GMM_OK;
}

gmm_status gmm_kernel_timer_end(double *ms, int64_t cap, int64_t *regions) {
    if (!g_collect) return GMM_ERR_INVALID_ARG;
    if ((cap > 0 && !ms) || cap < 0) return GMM_ERR_INVALID_ARG;
    g_collect = false;
    const size_t n = g_pairs_used;
    g_pairs_used = 0;
    if (regions) *regions = (int64_t)n;
    if (g_collect_failed) return GMM_ERR_CUDA;
    for (size_t i = 0; i < n; ++i) {
        if (cudaEventSynchronize(g_pool[2 * i + 1]) != cudaSuccess) return GMM_ERR_CUDA;
        float t = 0.f;
        if (cudaEventElapsedTime(&t, g_pool[2 * i], g_pool[2 * i + 1]) != cudaSuccess)
            return GMM_ERR_CUDA;
        if ((int64_t)i < cap) ms[i] = (double)t;
    }
    return GMM_OK;
}

gmm_status gmm_set_point_chunk(int64_t points) {
    if (points < 0) return GMM_ERR_INVALID_ARG;
    gmm_tc_set_chunk_override(points);
    return GMM_OK;
}

int64_t gmm_point_chunk(int64_t N, int d, int K, gmm_dtype dtype, uint32_t flags) {
    const int regime = gmm_regime(N, d, K, dtype, flags);
    if (regime < 0) return -1;
    return regime == 0 ? N : gmm_tc_chunk_points(N, d, K);
}

uint64_t gmm_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int gmm_device_binary_version(void) {
    cudaFuncAttributes a;
    if (gmm_kernel_attributes(&a) != cudaSuccess) {
        (void)cudaGetLastError();
        return -1;
    }
    return a.binaryVersion;
}

}  // extern "C"
