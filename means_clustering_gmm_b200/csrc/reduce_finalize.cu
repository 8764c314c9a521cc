// Deterministic cross-CTA reduction of the partial statistics and the M-step
// finalise.
//
// The SIMT kernels leave one fp32 partial of [K x (1+2d)] statistics per CTA
// (or per point range), the tensor-core kernels one fp64 partial per point
// range with S1 and S2 feature-major.  Their sum is taken here in fp64,
// partial by partial in slot order, so the result is bitwise reproducible
// run to run.  Where the pages' update adds each segment's sum into its
// centroid with a single atomic ("Flash-KMeans gor k-means realtime-venligt
// pa GPU ...", section "Centroid-opdatering uden atomics i stormvejr"), an
// ordered combine takes its place, identical in real arithmetic.
//
// Finalise: the textbook maximum-likelihood M-step of a diagonal GMM (the
// pages print no formula), in fp64:
//   N_k = S0_k, w_k = N_k / N, mu_kj = S1_kj / N_k,
//   var_kj = max(S2_kj / N_k - mu_kj^2, var_floor).
// A component with N_k < 1e-12 N keeps its mean and variance.
#include "common.cuh"
#include "kernels.h"

#include <math.h>

namespace gmmb {

// kFeatMajor: the partials hold S1 and S2 feature-major ([d][K], the layout
// the tensor-core kernels flush); the sum is written component-major.  The
// loop runs over the partials' own order so that their reads coalesce.
// accumulate: add the sum to what `stats` holds (a later point chunk of the
// same step) instead of writing it.
template <typename T, bool kFeatMajor>
__global__ void reduce_stats_kernel(const T *__restrict__ partial, int num_partials, int d, int K,
                                    double *__restrict__ stats, bool accumulate) {
    const int64_t width = (int64_t)K * (1 + 2 * (int64_t)d);
    const int64_t kd = (int64_t)K * d;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < width;
         i += (int64_t)gridDim.x * blockDim.x) {
        auto val = [&](int p) { return (double)partial[(size_t)p * width + i]; };
        // pairwise over slots in fixed 8-wide groups, then sequential: the
        // order depends only on num_partials
        double acc = 0.0;
        int p = 0;
        for (; p + 8 <= num_partials; p += 8) {
            double a0 = val(p) + val(p + 1), a1 = val(p + 2) + val(p + 3);
            double a2 = val(p + 4) + val(p + 5), a3 = val(p + 6) + val(p + 7);
            acc += (a0 + a1) + (a2 + a3);
        }
        for (; p < num_partials; ++p) acc += val(p);
        int64_t o = i;
        if (kFeatMajor && i >= K) {
            const int64_t j = i - K, half = j / kd, rem = j - half * kd;
            const int64_t f = rem / K, k = rem - f * K;
            o = K + half * kd + k * d + f;
        }
        stats[o] = accumulate ? stats[o] + acc : acc;
    }
}

// Single block: thread t sums a contiguous slice in order, then a fixed tree.
__global__ void __launch_bounds__(1024) reduce_ll_kernel(const double *__restrict__ part,
                                                         int64_t n, double *__restrict__ out,
                                                         bool accumulate) {
    __shared__ double sh[1024];
    const int t = threadIdx.x;
    int64_t per = (n + 1023) / 1024;
    int64_t b = t * per, e = b + per < n ? b + per : n;
    double acc = 0.0;
    for (int64_t i = b; i < e; ++i) acc += part[i];
    sh[t] = acc;
    __syncthreads();
    for (int s = 512; s; s >>= 1) {
        if (t < s) sh[t] += sh[t + s];
        __syncthreads();
    }
    if (t == 0) *out = accumulate ? *out + sh[0] : sh[0];
}

// One problem per blockIdx.y (batched GMM: problem b's statistics and
// parameters at b times the per-problem sizes; gridDim.y = 1 otherwise).
__global__ void finalize_kernel(const double *__restrict__ stats, int64_t N, int d, int K,
                                float var_floor, float *__restrict__ means,
                                float *__restrict__ vars, float *__restrict__ logw, int *err) {
    const size_t b = blockIdx.y;
    stats += b * (size_t)K * (1 + 2 * (size_t)d);
    means += b * (size_t)K * d;
    vars += b * (size_t)K * d;
    logw += b * (size_t)K;
    const double degenerate = 1e-12 * (double)N;
    const double *S0 = stats;
    const double *S1 = stats + K;
    const double *S2 = stats + K + (size_t)K * d;
    int64_t total = (int64_t)K * d;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        int k = (int)(i / d);
        double nk = S0[k];
        if (nk >= degenerate && nk > 0.0) {
            double mu = S1[i] / nk;
            double v = S2[i] / nk - mu * mu;
            if (v < (double)var_floor) v = (double)var_floor;
            float muf = (float)mu, vf = (float)v;
            if (!isfinite(muf) || !isfinite(vf)) set_error(err, GMM_ERR_NONFINITE);
            means[i] = muf;
            vars[i] = vf;
        }
        if (i % d == 0) {
            double lw = log(nk / (double)N);
            if (isnan(lw)) set_error(err, GMM_ERR_NONFINITE);
            logw[k] = (float)lw;
        }
    }
}

template <typename T, bool kFeatMajor>
static cudaError_t reduce_stats_t(const T *partial, int num_partials, int d, int K, double *stats,
                                  bool accumulate, cudaStream_t s) {
    const int64_t width = (int64_t)K * (1 + 2 * (int64_t)d);
    int64_t blocks = (width + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    reduce_stats_kernel<T, kFeatMajor><<<(unsigned)blocks, 256, 0, s>>>(partial, num_partials, d,
                                                                         K, stats, accumulate);
    return cudaGetLastError();
}

cudaError_t launch_reduce_stats(const float *partial, int num_partials, int d, int K,
                                double *stats, cudaStream_t s) {
    return reduce_stats_t<float, false>(partial, num_partials, d, K, stats, false, s);
}

cudaError_t launch_reduce_stats64(const double *partial, int num_partials, int d, int K,
                                  double *stats, bool accumulate, cudaStream_t s) {
    return reduce_stats_t<double, true>(partial, num_partials, d, K, stats, accumulate, s);
}

cudaError_t launch_reduce_ll(const double *ll_part, int64_t n, double *out, bool accumulate,
                             cudaStream_t s) {
    reduce_ll_kernel<<<1, 1024, 0, s>>>(ll_part, n, out, accumulate);
    return cudaGetLastError();
}

cudaError_t launch_finalize(const double *stats, int64_t N, int d, int K, float var_floor,
                            float *means, float *vars, float *logw, int *err, cudaStream_t s) {
    int64_t total = (int64_t)K * d;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    finalize_kernel<<<(unsigned)blocks, 256, 0, s>>>(stats, N, d, K, var_floor, means, vars,
                                                     logw, err);
    return cudaGetLastError();
}

cudaError_t launch_finalize_batched(const double *stats, int B, int64_t N, int d, int K,
                                    float var_floor, float *means, float *vars, float *logw,
                                    int *err, cudaStream_t s) {
    int64_t total = (int64_t)K * d;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    finalize_kernel<<<dim3((unsigned)blocks, (unsigned)B), 256, 0, s>>>(
        stats, N, d, K, var_floor, means, vars, logw, err);
    return cudaGetLastError();
}

cudaError_t gmm_kernel_attributes(cudaFuncAttributes *a) {
    return cudaFuncGetAttributes(a, finalize_kernel);
}

}  // namespace gmmb
