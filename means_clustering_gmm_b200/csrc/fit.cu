// The on-device EM fit loop and the k-means initialiser of a GMM fit.
//
// gmm_fit: EM iterations (gmm_em_step, then gmm_finalize) until the total
// log-likelihood stops improving, with the convergence test on the device.
// The loop is one CUDA graph: a reset kernel, then a conditional WHILE node
// whose body is one EM iteration followed by a one-thread control kernel
// that compares L_t with L_{t-1} and sets the loop condition.  The host
// launches the graph once and never waits inside the loop; it reads the
// outcome (iterations done, converged) once, at the end, from device memory.
// A soft clustering that stands in for k-means ("Flash-GMM: a
// memory-efficient kernel for scalable soft clustering", abstract: a drop-in
// replacement for k-means) is typically fitted this way, from a k-means
// start.
//
// gmm_init_kmeans: Lloyd iterations (kmeans_step, B = 1), then the GMM
// parameters of the final hard partition -- the maximum-likelihood M-step
// with responsibilities 0/1: member means, member variances (two-pass),
// weights count / N.
#include "common.cuh"
#include "kernels.h"

#include <math.h>

namespace gmmb {

namespace {

// Loop state of one fit, in the fit block of the workspace.
struct FitCtl {
    double L_prev;   // total log-likelihood of the previous iteration
    double L_cur;    // written by this iteration's gmm_em_step
    int iter;        // iterations done
    int converged;   // the last test met the tolerance
};

__global__ void fit_reset_kernel(FitCtl *c, int *info) {
    c->L_prev = -INFINITY;
    c->L_cur = -INFINITY;
    c->iter = 0;
    c->converged = 0;
    if (info) { info[0] = 0; info[1] = 0; }
}

// After iteration t's E-step (L_cur = L(theta_t)) and M-step: record L_t,
// test |L_t - L_{t-1}| <= tol |L_t|, and keep looping unless the test passed,
// max_iters is reached, a device error was recorded or L_t is not finite.
__global__ void fit_control_kernel(cudaGraphConditionalHandle h, FitCtl *c, int max_iters,
                                   double tol, double *trace, int *info, const int *err) {
    const int it = c->iter;
    const double L = c->L_cur;
    if (trace) trace[it] = L;
    const bool conv = it > 0 && fabs(L - c->L_prev) <= tol * fabs(L);
    const bool stop = conv || it + 1 >= max_iters || *(volatile const int *)err != 0 ||
                      !isfinite(L);
    c->L_prev = L;
    c->iter = it + 1;
    c->converged = conv ? 1 : 0;
    if (info) { info[0] = it + 1; info[1] = conv ? 1 : 0; }
    cudaGraphSetConditional(h, stop ? 0u : 1u);
}

// Weights of the hard partition: w_k = max(count_k, 1) / (N + empty), so an
// empty cluster keeps a one-point weight (it stays a live component with its
// centroid as mean and unit variance) and the weights sum to one.
__global__ void __launch_bounds__(1024) init_weights_kernel(const int32_t *__restrict__ counts,
                                                            int K, int64_t N,
                                                            float *__restrict__ logw) {
    __shared__ int part[1024];
    const int t = threadIdx.x;
    int e = 0;
    for (int k = t; k < K; k += 1024) e += counts[k] == 0;
    part[t] = e;
    __syncthreads();
    for (int o = 512; o; o >>= 1) {
        if (t < o) part[t] += part[t + o];
        __syncthreads();
    }
    const double denom = (double)N + (double)part[0];
    for (int k = t; k < K; k += 1024) {
        const int c = counts[k] > 0 ? counts[k] : 1;
        logw[k] = (float)log((double)c / denom);
    }
}

struct FitLayout {
    size_t em, stats, ctl, total;
};

FitLayout fit_layout(int64_t N, int d, int K, gmm_dtype dt) {
    FitLayout L;
    L.em = gmm_workspace_size(N, d, K, dt);
    L.stats = align_up(L.em);
    L.ctl = align_up(L.stats + sizeof(double) * (size_t)K * (1 + 2 * (size_t)d));
    L.total = align_up(L.ctl + sizeof(FitCtl));
    return L;
}

bool aligned_to(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

}  // namespace

}  // namespace gmmb

using namespace gmmb;

extern "C" size_t gmm_fit_workspace_size(int64_t N, int d, int K, gmm_dtype dtype) {
    if (gmm_workspace_size(N, d, K, dtype) == 0) return 0;
    return fit_layout(N, d, K, dtype).total;
}

extern "C" gmm_status gmm_fit(const void *X, gmm_dtype dtype, int64_t N, int d, int K,
                              float *means, float *vars, float *logw, int max_iters, double tol,
                              float var_floor, double *loglik_trace, int *fit_info, void *ws,
                              size_t ws_bytes, uint32_t flags, void *stream) {
    if (gmm_fit_workspace_size(N, d, K, dtype) == 0) return GMM_ERR_INVALID_ARG;
    const FitLayout L = fit_layout(N, d, K, dtype);
    if (ws_bytes < L.total || max_iters < 1 || !(tol >= 0.0) || !(var_floor > 0.f))
        return GMM_ERR_INVALID_ARG;
    if ((loglik_trace && !aligned_to(loglik_trace, 8)) || (fit_info && !aligned_to(fit_info, 4)))
        return GMM_ERR_INVALID_ARG;
    char *base = (char *)ws;
    double *stats = (double *)(base + L.stats);
    FitCtl *ctl = (FitCtl *)(base + L.ctl);
    // every argument check of the step itself, before anything is built
    const gmm_status chk = gmm_em_step_check(X, dtype, N, d, K, means, vars, logw, stats, nullptr,
                                             &ctl->L_cur, ws, L.em, flags);
    if (chk != GMM_OK) return chk;
    if (!means || !vars || !logw) return GMM_ERR_INVALID_ARG;

    cudaStream_t user = (cudaStream_t)stream;
    cudaStream_t cap = nullptr;
    cudaGraph_t g = nullptr;
    cudaGraphExec_t exec = nullptr;
    gmm_status rc = GMM_ERR_CUDA;
    // the kernel timer records events, which a conditional body cannot hold
    const bool was_suspended = timer_suspend(true);
    do {
        if (cudaStreamCreateWithFlags(&cap, cudaStreamNonBlocking) != cudaSuccess) break;
        if (cudaGraphCreate(&g, 0) != cudaSuccess) break;
        // reset node
        cudaGraphNode_t reset = nullptr;
        {
            void *args[] = {(void *)&ctl, (void *)&fit_info};
            cudaKernelNodeParams kp = {};
            kp.func = (void *)fit_reset_kernel;
            kp.gridDim = dim3(1);
            kp.blockDim = dim3(1);
            kp.kernelParams = args;
            if (cudaGraphAddKernelNode(&reset, g, nullptr, 0, &kp) != cudaSuccess) break;
        }
        // WHILE node, condition 1 at launch
        cudaGraphConditionalHandle h;
        if (cudaGraphConditionalHandleCreate(&h, g, 1, cudaGraphCondAssignDefault) != cudaSuccess)
            break;
        cudaGraphNodeParams cp = {};
        cp.type = cudaGraphNodeTypeConditional;
        cp.conditional.handle = h;
        cp.conditional.type = cudaGraphCondTypeWhile;
        cp.conditional.size = 1;
        cudaGraphNode_t loop = nullptr;
        if (cudaGraphAddNode(&loop, g, &reset, 1, &cp) != cudaSuccess) break;
        cudaGraph_t body = cp.conditional.phGraph_out[0];
        // the body: one EM iteration and the control kernel, captured
        if (cudaStreamBeginCaptureToGraph(cap, body, nullptr, nullptr, 0,
                                          cudaStreamCaptureModeRelaxed) != cudaSuccess)
            break;
        gmm_status st = gmm_em_step(X, dtype, N, d, K, means, vars, logw, stats, nullptr,
                                    &ctl->L_cur, ws, L.em, flags, (void *)cap);
        if (st == GMM_OK)
            st = gmm_finalize(stats, N, d, K, var_floor, means, vars, logw, ws, L.em,
                              (void *)cap);
        if (st == GMM_OK) {
            fit_control_kernel<<<1, 1, 0, cap>>>(h, ctl, max_iters, tol, loglik_trace, fit_info,
                                                 (const int *)ws);
            note_launches(1);
            if (cudaGetLastError() != cudaSuccess) st = GMM_ERR_CUDA;
        }
        cudaGraph_t captured = nullptr;
        const cudaError_t ec = cudaStreamEndCapture(cap, &captured);
        if (st != GMM_OK) { rc = st; break; }
        if (ec != cudaSuccess) break;
        if (cudaGraphInstantiate(&exec, g, 0) != cudaSuccess) break;
        if (cudaGraphLaunch(exec, user) != cudaSuccess) break;
        rc = GMM_OK;
    } while (0);
    timer_suspend(was_suspended);
    (void)cudaGetLastError();
    // an executable graph in flight is released when it completes
    if (exec) cudaGraphExecDestroy(exec);
    if (g) cudaGraphDestroy(g);
    if (cap) cudaStreamDestroy(cap);
    return rc;
}

// ------------------------------------------------------- k-means initialiser

extern "C" size_t gmm_init_kmeans_workspace_size(int64_t N, int d, int K) {
    const size_t km = kmeans_workspace_size(1, N, d, K);
    if (km == 0) return 0;
    // k-means workspace | second centroid buffer [K x d] | ids [N] | counts [K]
    return align_up(km) + align_up(sizeof(float) * (size_t)K * d) +
           align_up(sizeof(int32_t) * (size_t)N) + align_up(sizeof(int32_t) * (size_t)K);
}

extern "C" gmm_status gmm_init_kmeans(const void *X, gmm_dtype dtype, int64_t N, int d, int K,
                                      int iters, float var_floor, float *means, float *vars,
                                      float *logw, int32_t *ids, void *ws, size_t ws_bytes,
                                      void *stream) {
    const size_t need = gmm_init_kmeans_workspace_size(N, d, K);
    if (need == 0 || ws_bytes < need || iters < 1 || !(var_floor > 0.f)) return GMM_ERR_INVALID_ARG;
    if (!X || !means || !vars || !logw || !ws) return GMM_ERR_INVALID_ARG;
    if (!aligned_to(X, 16) || !aligned_to(ws, kAlign) || !aligned_to(means, 4) ||
        !aligned_to(vars, 4) || !aligned_to(logw, 4) || (ids && !aligned_to(ids, 4)))
        return GMM_ERR_INVALID_ARG;
    if (dtype != GMM_F32 && dtype != GMM_BF16 && dtype != GMM_F16) return GMM_ERR_INVALID_ARG;
    const size_t km = kmeans_workspace_size(1, N, d, K);
    char *b = (char *)ws;
    float *cbuf = (float *)(b + align_up(km));
    int32_t *ids_ws = (int32_t *)(b + align_up(km) + align_up(sizeof(float) * (size_t)K * d));
    int32_t *counts = (int32_t *)((char *)ids_ws + align_up(sizeof(int32_t) * (size_t)N));
    int32_t *id_out = ids ? ids : ids_ws;
    cudaStream_t s = (cudaStream_t)stream;
    // Lloyd iterations, centroids ping-ponging between `means` and cbuf;
    // the last one leaves the member means of the final partition in `means`
    float *cur = means, *nxt = cbuf;
    if (iters % 2 == 1) {   // start from the copy so that the last step writes `means`
        if (cudaMemcpyAsync(cbuf, means, sizeof(float) * (size_t)K * d, cudaMemcpyDeviceToDevice,
                            s) != cudaSuccess)
            return GMM_ERR_CUDA;
        cur = cbuf;
        nxt = means;
    }
    for (int t = 0; t < iters; ++t) {
        const gmm_status st = kmeans_step(X, dtype, 1, N, d, K, cur, id_out, nxt, counts, nullptr,
                                          ws, km, 0, stream);
        if (st != GMM_OK) return st;
        float *tmp = cur;
        cur = nxt;
        nxt = tmp;
    }
    // cur == means: member means of the last partition
    cudaError_t e = launch_km_member_vars(X, dtype, N, d, K, ws, means, var_floor, vars, s);
    if (e != cudaSuccess) return GMM_ERR_CUDA;
    init_weights_kernel<<<1, 1024, 0, s>>>(counts, K, N, logw);
    note_launches(1);
    return cudaGetLastError() == cudaSuccess ? GMM_OK : GMM_ERR_CUDA;
}
