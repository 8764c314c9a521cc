// gmm_em_step_static: the fused EM step with its workspace in a static device
// array instead of a caller buffer, for callers that cannot allocate device
// memory and hold no workspace (a plain C caller with only its input and
// output buffers and a fixed device-memory footprint: cudaMalloc / cudaFree
// on its path could fail under memory pressure and synchronise the device).
//
// The scratch is a file-scope __device__ array of GMM_STATIC_SCRATCH_BYTES,
// created with the module; its address is looked up once per device
// (cudaGetSymbolAddress, device current) on the first call and cached.  The
// call clears the error word (the only workspace field that must start at
// zero: every other field is fully written by the kernels before it is
// read), runs the ordinary gmm_em_step on the scratch, and copies the error
// word out.  Nothing here allocates.  All calls on a device share the one
// scratch, so calls whose device work overlaps in time race.
#include "common.cuh"
#include "kernels.h"

#include <mutex>

namespace {

static __device__ __align__(256) unsigned char g_scratch[GMM_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// The scratch's device address on the current device; set up on first use.
gmm_status scratch_for_current_device(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GMM_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GMM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) {
            (void)cudaGetLastError();
            return GMM_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return GMM_OK;
}

}  // namespace

extern "C" gmm_status gmm_em_step_static(const void *X, gmm_dtype dtype, int64_t N, int d, int K,
                                         const float *means, const float *vars,
                                         const float *logw, double *stats, float *loglik,
                                         double *loglik_total, int *device_status,
                                         uint32_t flags, void *stream) {
    const size_t need = gmm_workspace_size(N, d, K, dtype);
    if (need == 0) return GMM_ERR_INVALID_ARG;
    if (need > GMM_STATIC_SCRATCH_BYTES) return GMM_ERR_UNSUPPORTED;
    if (device_status && ((uintptr_t)device_status % sizeof(int)) != 0) return GMM_ERR_INVALID_ARG;
    void *ws = nullptr;
    const gmm_status st = scratch_for_current_device(&ws);
    if (st != GMM_OK) return st;
    // every argument check before the first write to the shared scratch: a
    // rejected call leaves the scratch (and any call in flight on it) alone
    const gmm_status chk = gmmb::gmm_em_step_check(X, dtype, N, d, K, means, vars, logw, stats,
                                                   loglik, loglik_total, ws,
                                                   GMM_STATIC_SCRATCH_BYTES, flags);
    if (chk != GMM_OK) return chk;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemsetAsync(ws, 0, sizeof(int), s) != cudaSuccess) return GMM_ERR_CUDA;
    const gmm_status r = gmm_em_step(X, dtype, N, d, K, means, vars, logw, stats, loglik,
                                     loglik_total, ws, GMM_STATIC_SCRATCH_BYTES, flags, stream);
    if (r != GMM_OK) return r;
    if (device_status &&
        cudaMemcpyAsync(device_status, ws, sizeof(int), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return GMM_ERR_CUDA;
    return GMM_OK;
}
