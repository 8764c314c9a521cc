// CUDA-core (SIMT) kernels of the GMM E-step, in the two-sweep form that the
// Flash-GMM design uses ("Turbo-GMM: FlashAttention-Inspired GPU-Accelerated
// Gaussian Mixture Model", abstract: the released Flash-GMM traverses the
// component dimension twice -- once for the normalisers, once to recompute
// the scores and accumulate the sufficient statistics).
//
//   sweep 1 (gmm_simt_lse_kernel):  l_n = LSE_k s_nk with an online max/sum
//                                   over component chunks; writes l_n.
//   sweep 2 (gmm_simt_stats_kernel): per (component chunk, point range),
//                                   recompute s_nk, r_nk = exp(s_nk - l_n),
//                                   accumulate S0/S1/S2 partials (fp32).
//
// Scores use the direct form s_nk = c_k + sum_j nhl_kj (x_nj - mu_kj)^2 with
// nhl = -1/(2 var) and c_k = log w_k - 1/2 sum_j log(2 pi var_kj), so no
// cancellation enters the CUDA-core path.  These kernels serve shapes the
// tensor-core kernels do not take and the GMM_FLAG_FORCE_SIMT test path.
#include "common.cuh"
#include "kernels.h"

#include <math.h>

namespace gmmb {

// a1 (CUDA-core form): nhl_kj = -1/(2 var_kj), c_k = log w_k - 1/2 sum_j log(2 pi var_kj).
// One warp per component; the fp64 sum over j runs in a fixed butterfly order.
// A mean or variance that is not finite, a variance <= 0 or a log weight that
// is NaN or +inf records GMM_ERR_NONFINITE.
__global__ void gmm_simt_precompute_kernel(const float *__restrict__ means,
                                           const float *__restrict__ vars,
                                           const float *__restrict__ logw, int K, int d,
                                           float *__restrict__ nhl, float *__restrict__ ck,
                                           int *err) {
    int warp = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5);
    int lane = threadIdx.x & 31;
    if (warp >= K) return;
    double acc = 0.0;
    bool bad = lane == 0 && (isnan(logw[warp]) || logw[warp] == INFINITY);
    for (int j = lane; j < d; j += 32) {
        float v = vars[(size_t)warp * d + j];
        bad |= !isfinite(means[(size_t)warp * d + j]) || !isfinite(v) || !(v > 0.f);
        nhl[(size_t)warp * d + j] = -0.5f / v;
        acc += log(2.0 * M_PI * (double)v);
    }
    if (bad) set_error(err, GMM_ERR_NONFINITE);
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) ck[warp] = (float)((double)logw[warp] - 0.5 * acc);
}

// Sweep 1.  Block = 256 threads = 16 (component lanes tx) x 16 (point rows ty);
// each thread owns a 4-point x 4-component micro tile of a 64 x 64 score tile.
template <typename T>
__global__ void __launch_bounds__(256)
gmm_simt_lse_kernel(const T *__restrict__ X, int64_t N, int d, int K,
                    const float *__restrict__ means, const float *__restrict__ nhl,
                    const float *__restrict__ ck, float *__restrict__ lse,
                    float *__restrict__ loglik, double *__restrict__ ll_part, int *err) {
    constexpr int TP = kLseTileP, TK = kLseTileK, TJ = kLseTileJ;
    __shared__ __align__(16) float Xs[TJ][TP + 4];
    __shared__ __align__(16) float Ms[TJ][TK + 4];
    __shared__ __align__(16) float Hs[TJ][TK + 4];
    __shared__ double lsum[TP];
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const int64_t ntiles = (N + TP - 1) / TP;

    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t p0 = tile * TP;
        float m[4], l[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) { m[i] = -INFINITY; l[i] = 0.f; }

        for (int k0 = 0; k0 < K; k0 += TK) {
            float acc[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[i][c] = 0.f;

            for (int j0 = 0; j0 < d; j0 += TJ) {
                __syncthreads();
                // stage X[p0.., j0..] transposed, and the mu / nhl chunk
                for (int e = tid; e < TP * TJ; e += 256) {
                    int pl = e / TJ, jl = e % TJ;
                    int64_t p = p0 + pl;
                    int j = j0 + jl;
                    Xs[jl][pl] = (p < N && j < d) ? load_elem<T>(X + p * d + j) : 0.f;
                }
                for (int e = tid; e < TK * TJ; e += 256) {
                    int kl = e / TJ, jl = e % TJ;
                    int k = k0 + kl, j = j0 + jl;
                    bool ok = (k < K && j < d);
                    Ms[jl][kl] = ok ? __ldg(means + (size_t)k * d + j) : 0.f;
                    Hs[jl][kl] = ok ? __ldg(nhl + (size_t)k * d + j) : 0.f;
                }
                __syncthreads();
#pragma unroll 4
                for (int jl = 0; jl < TJ; ++jl) {
                    float4 xv = *reinterpret_cast<const float4 *>(&Xs[jl][ty * 4]);
                    float4 mv = *reinterpret_cast<const float4 *>(&Ms[jl][tx * 4]);
                    float4 hv = *reinterpret_cast<const float4 *>(&Hs[jl][tx * 4]);
                    float xs[4] = {xv.x, xv.y, xv.z, xv.w};
                    float ms[4] = {mv.x, mv.y, mv.z, mv.w};
                    float hs[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            float df = xs[i] - ms[c];
                            acc[i][c] = fmaf(df * df, hs[c], acc[i][c]);
                        }
                }
            }
            // add the per-component constant; mask components beyond K
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                int k = k0 + tx * 4 + c;
                float cc = k < K ? __ldg(ck + k) : -INFINITY;
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i][c] = (k < K) ? acc[i][c] + cc : -INFINITY;
            }
            // online LSE over this chunk; the 16 lanes of a point row share it
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float cm = fmaxf(fmaxf(acc[i][0], acc[i][1]), fmaxf(acc[i][2], acc[i][3]));
#pragma unroll
                for (int o = 8; o; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
                float nm = fmaxf(m[i], cm);
                float cs = 0.f;
                if (nm != -INFINITY) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) cs += __expf(acc[i][c] - nm);
                }
#pragma unroll
                for (int o = 8; o; o >>= 1) cs += __shfl_xor_sync(0xffffffffu, cs, o);
                l[i] = (nm == -INFINITY) ? 0.f : l[i] * __expf(m[i] - nm) + cs;
                m[i] = nm;
            }
        }
        // write l_n = m + log(l)
        if (tx == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int pl = ty * 4 + i;
                int64_t p = p0 + pl;
                float v = m[i] + logf(l[i]);
                if (p < N) {
                    if (!(m[i] > -INFINITY)) set_error(err, GMM_ERR_NONFINITE);
                    lse[p] = v;
                    if (loglik) loglik[p] = v;
                    lsum[pl] = (double)v;
                } else {
                    lsum[pl] = 0.0;
                }
            }
        }
        __syncthreads();
        if (tid < 32) {  // fixed-order sum of the tile's 64 values
            double s = lsum[tid] + lsum[tid + 32];
#pragma unroll
            for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (tid == 0) ll_part[tile] = s;
        }
    }
}

// Sweep 2.  Block = 256 threads; the block owns `tk` components (tk * groups
// = 256 threads, 16 features per thread) and a contiguous range of points.
template <typename T>
__global__ void __launch_bounds__(256)
gmm_simt_stats_kernel(const T *__restrict__ X, int64_t N, int d, int K, int tk, int groups,
                      int64_t range_pts, const float *__restrict__ means,
                      const float *__restrict__ nhl, const float *__restrict__ ck,
                      const float *__restrict__ lse, float *__restrict__ partial) {
    extern __shared__ __align__(16) float smem[];
    constexpr int TP = kStatsTileP;
    const int dp = groups * 16;           // padded feature count
    const int xs_stride = dp + 4;
    float *Xs = smem;                     // [TP][xs_stride]
    float *Ms = Xs + TP * xs_stride;      // [tk][d + 1]
    float *Hs = Ms + tk * (d + 1);        // [tk][d + 1]
    float *Rs = Hs + tk * (d + 1);        // [TP][tk + 1]
    float *Ls = Rs + TP * (tk + 1);       // [TP]
    float *Cs = Ls + TP;                  // [tk]

    const int tid = threadIdx.x;
    const int k0 = blockIdx.x * tk;
    const int64_t pbeg = (int64_t)blockIdx.y * range_pts;
    const int64_t pend = min(N, pbeg + range_pts);

    for (int e = tid; e < tk * d; e += 256) {
        int kl = e / d, j = e % d;
        int k = k0 + kl;
        Ms[kl * (d + 1) + j] = k < K ? __ldg(means + (size_t)k * d + j) : 0.f;
        Hs[kl * (d + 1) + j] = k < K ? __ldg(nhl + (size_t)k * d + j) : 0.f;
    }
    for (int e = tid; e < tk; e += 256) Cs[e] = (k0 + e < K) ? __ldg(ck + k0 + e) : -INFINITY;

    const int kk = tid / groups;       // component owned in the accumulation
    const int g = tid % groups;        // feature group owned
    const bool acc_active = kk < tk;
    float s0 = 0.f, s1[16], s2[16];
#pragma unroll
    for (int f = 0; f < 16; ++f) { s1[f] = 0.f; s2[f] = 0.f; }

    for (int64_t p0 = pbeg; p0 < pend; p0 += TP) {
        __syncthreads();
        for (int e = tid; e < TP * dp; e += 256) {
            int pl = e / dp, j = e % dp;
            int64_t p = p0 + pl;
            Xs[pl * xs_stride + j] = (p < pend && j < d) ? load_elem<T>(X + p * d + j) : 0.f;
        }
        for (int e = tid; e < TP; e += 256) {
            int64_t p = p0 + e;
            Ls[e] = p < pend ? lse[p] : INFINITY;  // INFINITY -> r = 0 for padding rows
        }
        __syncthreads();
        // scores and responsibilities for TP x tk pairs
        for (int e = tid; e < TP * tk; e += 256) {
            int pl = e / tk, kl = e % tk;
            const float *xr = Xs + pl * xs_stride;
            const float *mr = Ms + kl * (d + 1);
            const float *hr = Hs + kl * (d + 1);
            float acc = 0.f;
            for (int j = 0; j < d; ++j) {
                float df = xr[j] - mr[j];
                acc = fmaf(df * df, hr[j], acc);
            }
            float s = acc + Cs[kl];
            float r = (Cs[kl] == -INFINITY) ? 0.f : __expf(s - Ls[pl]);
            Rs[pl * (tk + 1) + kl] = r;
        }
        __syncthreads();
        if (acc_active) {
            for (int pl = 0; pl < TP; ++pl) {
                float r = Rs[pl * (tk + 1) + kk];
                const float *xr = Xs + pl * xs_stride + g * 16;
                s0 += r;
#pragma unroll
                for (int f = 0; f < 16; f += 4) {
                    float4 xv = *reinterpret_cast<const float4 *>(xr + f);
                    float rx0 = r * xv.x, rx1 = r * xv.y, rx2 = r * xv.z, rx3 = r * xv.w;
                    s1[f] += rx0; s1[f + 1] += rx1; s1[f + 2] += rx2; s1[f + 3] += rx3;
                    s2[f] = fmaf(rx0, xv.x, s2[f]);
                    s2[f + 1] = fmaf(rx1, xv.y, s2[f + 1]);
                    s2[f + 2] = fmaf(rx2, xv.z, s2[f + 2]);
                    s2[f + 3] = fmaf(rx3, xv.w, s2[f + 3]);
                }
            }
        }
    }
    // write this block's partial statistics (only its components)
    if (acc_active) {
        int k = k0 + kk;
        if (k < K) {
            float *out = partial + (size_t)blockIdx.y * ((size_t)K * (1 + 2 * (size_t)d));
            if (g == 0) out[k] = s0;
#pragma unroll
            for (int f = 0; f < 16; ++f) {
                int j = g * 16 + f;
                if (j < d) {
                    out[K + (size_t)k * d + j] = s1[f];
                    out[K + (size_t)K * d + (size_t)k * d + j] = s2[f];
                }
            }
        }
    }
}

size_t gmm_simt_stats_smem(int d, int tk, int groups) {
    int dp = groups * 16;
    return sizeof(float) * ((size_t)kStatsTileP * (dp + 4) + 2 * (size_t)tk * (d + 1) +
                            (size_t)kStatsTileP * (tk + 1) + kStatsTileP + tk);
}

template <typename T>
static cudaError_t launch_simt_t(const T *X, int64_t N, int d, int K, const float *means,
                                 const float *vars, const float *logw, const GmmWs &w,
                                 float *loglik, cudaStream_t s) {
    GmmSimtPlan p = gmm_simt_plan(N, d, K);
    int pre_blocks = (K * 32 + 255) / 256;
    gmm_simt_precompute_kernel<<<pre_blocks, 256, 0, s>>>(means, vars, logw, K, d, w.nhl, w.ck,
                                                          w.err);
    int64_t g1 = p.lse_tiles < (1 << 20) ? p.lse_tiles : (1 << 20);
    timer_begin(s);
    gmm_simt_lse_kernel<T><<<(unsigned)g1, 256, 0, s>>>(X, N, d, K, means, w.nhl, w.ck, w.lse,
                                                        loglik, w.ll_part, w.err);
    size_t smem = gmm_simt_stats_smem(d, p.tk, p.groups);
    cudaError_t e = cudaFuncSetAttribute(gmm_simt_stats_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.kchunks, p.ranges);
    gmm_simt_stats_kernel<T><<<grid, 256, smem, s>>>(X, N, d, K, p.tk, p.groups, p.range_pts,
                                                     means, w.nhl, w.ck, w.lse, w.partial);
    timer_end(s);
    note_launches(3);
    return cudaGetLastError();
}

// Soft assignment on CUDA cores (shapes without a tensor-core kernel): one
// thread per point, components staged through shared memory in chunks;
// direct-form scores s = c_k + sum_j nhl_kj (x_j - mu_kj)^2, an online
// (max, sum) for l_n and the top-kTopMax (score, id) list; then
// r = exp(s - l_n) for the first R entries, cut at tau.
constexpr int kAsgThreads = 128;
constexpr int kAsgSmem = 48 * 1024;

template <typename T>
__global__ void __launch_bounds__(kAsgThreads)
gmm_simt_assign_kernel(const T *__restrict__ X, int64_t N, int d, int K,
                       const float *__restrict__ means, const float *__restrict__ nhl,
                       const float *__restrict__ ck, float *__restrict__ lse_out,
                       float *__restrict__ loglik, int R, float tau, int32_t *__restrict__ ids,
                       float *__restrict__ resp, int *err) {
    extern __shared__ float sh[];
    const int kc = (kAsgSmem / 4) / (2 * d + 1);   // components per chunk
    float *smu = sh, *snhl = sh + (size_t)kc * d, *sck = sh + 2 * (size_t)kc * d;
    const int64_t n = blockIdx.x * (int64_t)kAsgThreads + threadIdx.x;
    const bool valid = n < N;
    const T *xr = X + (valid ? n : 0) * d;
    float m = -INFINITY, l = 0.f;
    float ts[kTopMax];
    int ti[kTopMax];
#pragma unroll
    for (int j = 0; j < kTopMax; ++j) { ts[j] = -INFINITY; ti[j] = -1; }
    for (int k0 = 0; k0 < K; k0 += kc) {
        const int nk = min(kc, K - k0);
        __syncthreads();
        for (int i = threadIdx.x; i < nk * d; i += kAsgThreads) {
            smu[i] = means[(size_t)k0 * d + i];
            snhl[i] = nhl[(size_t)k0 * d + i];
        }
        for (int i = threadIdx.x; i < nk; i += kAsgThreads) sck[i] = ck[k0 + i];
        __syncthreads();
        if (!valid) continue;
        for (int c = 0; c < nk; ++c) {
            float acc = 0.f;
            for (int j = 0; j < d; ++j) {
                const float df = load_elem<T>(xr + j) - smu[c * d + j];
                acc = fmaf(snhl[c * d + j] * df, df, acc);
            }
            const float sc = sck[c] + acc;
            if (sc > m) {
                l = (m == -INFINITY ? 0.f : l * expf(m - sc)) + 1.f;
                m = sc;
            } else if (sc > -INFINITY) {
                l += expf(sc - m);
            }
            if (sc > ts[kTopMax - 1]) topr_insert(ts, ti, sc, k0 + c);
        }
    }
    if (!valid) return;
    const float lse = m + logf(l);
    if (!(m > -INFINITY)) set_error(err, GMM_ERR_NONFINITE);
    lse_out[n] = lse;
    if (loglik) loglik[n] = lse;
#pragma unroll
    for (int j = 0; j < kTopMax; ++j) {
        if (j < R) {
            const float r = ti[j] >= 0 ? expf(ts[j] - lse) : 0.f;
            const bool keep = ti[j] >= 0 && r >= tau;
            ids[n * R + j] = keep ? ti[j] : -1;
            resp[n * R + j] = keep ? r : 0.f;
        }
    }
}

cudaError_t launch_gmm_simt_assign(const void *X, gmm_dtype dt, int64_t N, int d, int K,
                                   const float *means, const float *vars, const float *logw,
                                   const GmmWs &w, float *loglik, int R, float tau, int32_t *ids,
                                   float *resp, cudaStream_t s) {
    const int pre_blocks = (K * 32 + 255) / 256;
    gmm_simt_precompute_kernel<<<pre_blocks, 256, 0, s>>>(means, vars, logw, K, d, w.nhl, w.ck,
                                                          w.err);
    const unsigned grid = (unsigned)((N + kAsgThreads - 1) / kAsgThreads);
    switch (dt) {
        case GMM_F32:
            gmm_simt_assign_kernel<float><<<grid, kAsgThreads, kAsgSmem, s>>>(
                (const float *)X, N, d, K, means, w.nhl, w.ck, w.lse, loglik, R, tau, ids, resp,
                w.err);
            break;
        case GMM_BF16:
            gmm_simt_assign_kernel<__nv_bfloat16><<<grid, kAsgThreads, kAsgSmem, s>>>(
                (const __nv_bfloat16 *)X, N, d, K, means, w.nhl, w.ck, w.lse, loglik, R, tau, ids,
                resp, w.err);
            break;
        default:
            gmm_simt_assign_kernel<__half><<<grid, kAsgThreads, kAsgSmem, s>>>(
                (const __half *)X, N, d, K, means, w.nhl, w.ck, w.lse, loglik, R, tau, ids, resp,
                w.err);
    }
    note_launches(2);
    return cudaGetLastError();
}

cudaError_t launch_gmm_simt(const void *X, gmm_dtype dt, int64_t N, int d, int K,
                            const float *means, const float *vars, const float *logw,
                            const GmmWs &w, float *loglik, int *num_partials, int64_t *num_ll,
                            cudaStream_t s) {
    GmmSimtPlan p = gmm_simt_plan(N, d, K);
    *num_partials = p.ranges;
    *num_ll = p.lse_tiles;
    switch (dt) {
        case GMM_F32:
            return launch_simt_t<float>((const float *)X, N, d, K, means, vars, logw, w, loglik, s);
        case GMM_BF16:
            return launch_simt_t<__nv_bfloat16>((const __nv_bfloat16 *)X, N, d, K, means, vars,
                                                logw, w, loglik, s);
        case GMM_F16:
            return launch_simt_t<__half>((const __half *)X, N, d, K, means, vars, logw, w,
                                         loglik, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace gmmb
