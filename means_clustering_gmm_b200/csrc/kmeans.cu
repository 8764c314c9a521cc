// Lloyd k-means as the hard-assignment special case of the fused EM step.
//
// Assignment ("Flash-KMeans gor k-means realtime-venligt pa GPU ...", section
// "FlashAssign gor tildelingen hurtig"; "Hvorfor IO og ikke FLOPs bider"):
// point tiles and centroid tiles are streamed through on-chip memory, the
// distance of every pair is formed there and only a running (best distance,
// best index) per point is kept -- the N x K distance matrix is never
// written.  Ties go to the lowest centroid index (strict < in increasing k).
//
// Update (same article, "Centroid-opdatering uden atomics i stormvejr"; the
// zubnet.ai article on Flash-KMeans calls it an explicit inverse mapping with
// ordered segment reductions): a stable counting argsort of the ids gives
// contiguous segments per cluster; each segment's rows are gathered through
// the permutation (the point matrix is not moved) and summed in point order;
// centroid = sum / count, and an empty cluster keeps its centroid.  The sort
// is three passes -- per-chunk histograms, an exclusive scan, a stable
// scatter -- and nothing uses floating-point atomics, so the result is
// bitwise reproducible.
#include "common.cuh"
#include "kernels.h"
#include "kmeans_tc.h"

#include <type_traits>

namespace gmmb {

constexpr int kKmTileP = 64, kKmTileK = 64, kKmTileJ = 32;
constexpr int kSortChunk = 2048;  // points per sort chunk (8 warps x 256)

KmWsLayout km_ws_layout(int B, int64_t N, int d, int K) {
    KmWsLayout L;
    size_t o = kAlign;  // error word
    L.nblk = (int)((N + kSortChunk - 1) / kSortChunk);
    L.assign_tiles = (int)((N + kKmTileP - 1) / kKmTileP);
    int tc_tiles = km_tc_tiles_per_problem(N);
    if (tc_tiles > L.assign_tiles) L.assign_tiles = tc_tiles;
    L.off_mind = o;    o = align_up(o + sizeof(float) * (size_t)B * N);
    L.off_hist = o;    o = align_up(o + sizeof(int32_t) * (size_t)B * K * L.nblk);
    L.off_perm = o;    o = align_up(o + sizeof(int32_t) * (size_t)B * N);
    L.off_segoff = o;  o = align_up(o + sizeof(int32_t) * (size_t)B * (K + 1));
    L.off_inpart = o;  o = align_up(o + sizeof(double) * (size_t)B * L.assign_tiles);
    L.off_cnorm = o;   o = align_up(o + km_tc_param_bytes(B, d, K));
    L.off_segin = o;   o = align_up(o + sizeof(double) * (size_t)B * K);
    L.total = o;
    return L;
}

// ---------------------------------------------------------------- assign
// CUDA-core assignment: 64 points x 64 centroids per block tile, direct
// squared distances sum_j (x_j - c_j)^2, 4 x 4 micro tile per thread.
template <typename T>
__global__ void __launch_bounds__(256)
km_simt_assign_kernel(const T *__restrict__ X, int64_t N, int d, int K,
                      const float *__restrict__ C, int32_t *__restrict__ ids,
                      float *__restrict__ mind, double *__restrict__ inpart, int tiles_stride) {
    constexpr int TP = kKmTileP, TK = kKmTileK, TJ = kKmTileJ;
    __shared__ __align__(16) float Xs[TJ][TP + 4];
    __shared__ __align__(16) float Cs[TJ][TK + 4];
    __shared__ double dsum[TP];
    const int b = blockIdx.y;
    const T *Xb = X + (size_t)b * N * d;
    const float *Cb = C + (size_t)b * K * d;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int64_t p0 = (int64_t)blockIdx.x * TP;

    float best[4];
    int bidx[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) { best[i] = INFINITY; bidx[i] = 0; }

    for (int k0 = 0; k0 < K; k0 += TK) {
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[i][c] = 0.f;
        for (int j0 = 0; j0 < d; j0 += TJ) {
            __syncthreads();
            for (int e = tid; e < TP * TJ; e += 256) {
                int pl = e / TJ, jl = e % TJ;
                int64_t p = p0 + pl;
                int j = j0 + jl;
                Xs[jl][pl] = (p < N && j < d) ? load_elem<T>(Xb + p * d + j) : 0.f;
            }
            for (int e = tid; e < TK * TJ; e += 256) {
                int kl = e / TJ, jl = e % TJ;
                int k = k0 + kl, j = j0 + jl;
                Cs[jl][kl] = (k < K && j < d) ? __ldg(Cb + (size_t)k * d + j) : 0.f;
            }
            __syncthreads();
#pragma unroll 4
            for (int jl = 0; jl < TJ; ++jl) {
                float4 xv = *reinterpret_cast<const float4 *>(&Xs[jl][ty * 4]);
                float4 cv = *reinterpret_cast<const float4 *>(&Cs[jl][tx * 4]);
                float xs[4] = {xv.x, xv.y, xv.z, xv.w};
                float cs[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float df = xs[i] - cs[c];
                        acc[i][c] = fmaf(df, df, acc[i][c]);
                    }
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // best of this thread's 4 centroids (increasing k, strict <)
            float cb = INFINITY;
            int ci = 0x7fffffff;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                int k = k0 + tx * 4 + c;
                if (k < K && acc[i][c] < cb) { cb = acc[i][c]; ci = k; }
            }
            // across the 16 lanes of the point row: (distance, index) lexicographic
#pragma unroll
            for (int o = 8; o; o >>= 1) {
                float ob = __shfl_xor_sync(0xffffffffu, cb, o);
                int oi = __shfl_xor_sync(0xffffffffu, ci, o);
                if (ob < cb || (ob == cb && oi < ci)) { cb = ob; ci = oi; }
            }
            if (cb < best[i]) { best[i] = cb; bidx[i] = ci; }
        }
    }
    if (tx == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int pl = ty * 4 + i;
            int64_t p = p0 + pl;
            if (p < N) {
                ids[(size_t)b * N + p] = bidx[i];
                mind[(size_t)b * N + p] = best[i];
                dsum[pl] = (double)best[i];
            } else {
                dsum[pl] = 0.0;
            }
        }
    }
    __syncthreads();
    if (tid < 32) {
        double s = dsum[tid] + dsum[tid + 32];
#pragma unroll
        for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (tid == 0) inpart[(size_t)b * tiles_stride + blockIdx.x] = s;
    }
}

// ------------------------------------------------------------ sort-inverse
// Pass 1: per-chunk histogram of the ids, stored [b][k][chunk] so that an
// exclusive scan in that order yields, for every (k, chunk), the first slot of
// the chunk's members of cluster k.
__global__ void __launch_bounds__(256)
km_hist_kernel(const int32_t *__restrict__ ids, int64_t N, int K, int nblk,
               int32_t *__restrict__ hist) {
    extern __shared__ int32_t h[];
    const int b = blockIdx.y, blk = blockIdx.x;
    for (int k = threadIdx.x; k < K; k += 256) h[k] = 0;
    __syncthreads();
    const int64_t n0 = (int64_t)blk * kSortChunk;
    const int64_t n1 = min(N, n0 + kSortChunk);
    for (int64_t n = n0 + threadIdx.x; n < n1; n += 256) atomicAdd(&h[ids[(size_t)b * N + n]], 1);
    __syncthreads();
    for (int k = threadIdx.x; k < K; k += 256)
        hist[((size_t)b * K + k) * nblk + blk] = h[k];
}

// Pass 2: exclusive scan of [k][chunk] per problem (one 1024-thread block per
// problem), in place; also the segment starts segoff[b][k] and segoff[b][K]=N.
// Warp w owns the w-th of 32 contiguous ranges of the E = K * nblk entries
// (whole 32-entry rounds), so every load and store of a round is one
// coalesced 128-byte line: the warp sums its range, warp 0 scans the 32
// totals, and each warp then scans its rounds with shuffles, carrying the
// running prefix.  Integer sums: the result does not depend on the order.
template <typename I>
__global__ void __launch_bounds__(1024)
km_scan_kernel(int32_t *__restrict__ hist, int64_t N, int K, int nblk,
               int32_t *__restrict__ segoff) {
    __shared__ int32_t wsum[32];
    const int b = blockIdx.x, t = threadIdx.x, w = t >> 5, lane = t & 31;
    int32_t *h = hist + (size_t)b * K * nblk;
    const I E = (I)K * (I)nblk;
    const I per = ((E + 31) / 32 + 31) / 32 * 32;   // entries per warp, whole rounds
    const I e0 = (I)w * per;
    const I e1 = e0 + per < E ? e0 + per : E;
    int32_t s = 0;
    for (I e = e0 + lane; e < e1; e += 32) s += h[e];
    s = __reduce_add_sync(0xffffffffu, s);
    if (lane == 0) wsum[w] = s;
    __syncthreads();
    if (w == 0) {
        const int32_t own = wsum[lane];
        int32_t v = own;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t u = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += u;
        }
        wsum[lane] = v - own;   // exclusive prefix of warp `lane`'s range
    }
    __syncthreads();
    int32_t run = wsum[w];
    int32_t *so = segoff + (size_t)b * (K + 1);
    // eight rounds at a time: their loads are all issued before the stores
    // that rewrite the same array, so they overlap instead of waiting one by one
    constexpr int R = 8;
    for (I e = e0; e < e1; e += 32 * R) {
        int32_t c[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const I i = e + 32 * r + lane;
            c[r] = i < e1 ? h[i] : 0;
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const I i = e + 32 * r + lane;
            int32_t v = c[r];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            if (i < e1) {
                const int32_t excl = run + v - c[r];
                h[i] = excl;
                if (i % nblk == 0) so[i / nblk] = excl;
            }
            run += __shfl_sync(0xffffffffu, v, 31);
        }
    }
    if (t == 0) so[K] = (int32_t)N;
}

// Pass 3: stable scatter.  Each of the 8 warps owns 256 consecutive points of
// the chunk and walks them in rounds of 32; __match_any_sync groups equal ids
// within a round, so ranks follow point order without atomics.
__global__ void __launch_bounds__(256)
km_scatter_kernel(const int32_t *__restrict__ ids, int64_t N, int K, int nblk,
                  const int32_t *__restrict__ offs, int32_t *__restrict__ perm) {
    extern __shared__ int32_t cnt[];  // [8][K]
    const int b = blockIdx.y, blk = blockIdx.x;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < 8 * K; i += 256) cnt[i] = 0;
    __syncthreads();
    const int64_t base = (int64_t)blk * kSortChunk + (int64_t)w * (kSortChunk / 8);
    const unsigned lt = (1u << lane) - 1u;
    for (int r = 0; r < kSortChunk / 8 / 32; ++r) {
        int64_t n = base + r * 32 + lane;
        int key = n < N ? ids[(size_t)b * N + n] : -1;
        unsigned peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0 && lane == __ffs(peers) - 1) cnt[w * K + key] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    for (int k = threadIdx.x; k < K; k += 256) {
        int32_t run = 0;
        for (int ww = 0; ww < 8; ++ww) {
            int32_t c = cnt[ww * K + k];
            cnt[ww * K + k] = run;
            run += c;
        }
    }
    __syncthreads();
    for (int r = 0; r < kSortChunk / 8 / 32; ++r) {
        int64_t n = base + r * 32 + lane;
        int key = n < N ? ids[(size_t)b * N + n] : -1;
        unsigned peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0) {
            int32_t pos = offs[((size_t)b * K + key) * nblk + blk] + cnt[w * K + key] +
                          __popc(peers & lt);
            perm[(size_t)b * N + pos] = (int32_t)n;
        }
        __syncwarp();
        if (key >= 0 && lane == __ffs(peers) - 1) cnt[w * K + key] += __popc(peers);
        __syncwarp();
    }
}

// Segmented reduction: one warp per (problem, cluster) segment; members are
// read through the permutation in point order and summed in fp64.  The same
// pass adds up the members' squared distances to the centroid they were
// assigned to (fp64, direct form), the segment's share of the inertia.
template <typename T>
__global__ void __launch_bounds__(256)
km_segreduce_kernel(const T *__restrict__ X, int B, int64_t N, int d, int K,
                    const int32_t *__restrict__ perm, const int32_t *__restrict__ segoff,
                    const float *__restrict__ C, float *__restrict__ newC,
                    int32_t *__restrict__ counts, double *__restrict__ segin) {
    const int64_t seg = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (seg >= (int64_t)B * K) return;
    const int b = (int)(seg / K), k = (int)(seg % K);
    const int32_t s0 = segoff[(size_t)b * (K + 1) + k];
    const int32_t s1 = segoff[(size_t)b * (K + 1) + k + 1];
    const int32_t cnt = s1 - s0;
    if (counts && lane == 0) counts[seg] = cnt;
    const T *Xb = X + (size_t)b * N * d;
    double dist = 0.0;
    for (int jb = 0; jb < d; jb += 128) {
        double acc[4] = {0.0, 0.0, 0.0, 0.0};
        double cj[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            int j = jb + lane + 32 * t;
            cj[t] = j < d ? (double)C[((size_t)b * K + k) * d + j] : 0.0;
        }
        for (int32_t m = s0; m < s1; ++m) {
            const T *row = Xb + (size_t)perm[(size_t)b * N + m] * d;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                int j = jb + lane + 32 * t;
                if (j < d) {
                    const double x = (double)load_elem<T>(row + j);
                    acc[t] += x;
                    dist += (x - cj[t]) * (x - cj[t]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            int j = jb + lane + 32 * t;
            if (j < d) {
                size_t i = ((size_t)b * K + k) * d + j;
                newC[i] = cnt > 0 ? (float)(acc[t] / (double)cnt) : C[i];
            }
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) dist += __shfl_xor_sync(0xffffffffu, dist, o);
    if (lane == 0) segin[seg] = dist;
}

// The same segmented reduction for d = 64 or 128, with more rows in flight:
// the warp's lanes form 4 groups of 8; group g takes members m = s0 + g,
// s0 + g + 4, ... (two at a time), each lane holding D/8 consecutive features
// read with 16-byte loads.  Per lane: fp64 sums of x and of x^2 (two per
// element, and no centroid held in registers during the loop); the members'
// squared distance to the old centroid c follows at the end as
// sum x^2 - 2 c . sum x + n |c|^2, in fp64 (the fp16/fp32 inputs leave that
// form 2^-53-relative to sum x^2).  The 4 groups are combined in group order,
// so the result is reproducible.
template <typename T, int D>
__global__ void __launch_bounds__(256)
km_segreduce_vec_kernel(const T *__restrict__ X, int B, int64_t N, int K,
                        const int32_t *__restrict__ perm, const int32_t *__restrict__ segoff,
                        const float *__restrict__ C, float *__restrict__ newC,
                        int32_t *__restrict__ counts, double *__restrict__ segin) {
    constexpr int F = D / 8;                       // features per lane
    constexpr int VEC = 16 / sizeof(T);            // elements per 16-byte load
    static_assert(F % VEC == 0, "features per lane must fill whole 16-byte loads");
    const int64_t seg = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31, grp = lane >> 3, sub = lane & 7;
    if (seg >= (int64_t)B * K) return;
    const int b = (int)(seg / K), k = (int)(seg % K);
    const int32_t s0 = segoff[(size_t)b * (K + 1) + k];
    const int32_t s1 = segoff[(size_t)b * (K + 1) + k + 1];
    const int32_t cnt = s1 - s0;
    if (counts && lane == 0) counts[seg] = cnt;
    const T *Xb = X + (size_t)b * N * D;
    const int32_t *pb = perm + (size_t)b * N;
    const float *cr = C + ((size_t)b * K + k) * D + sub * F;
    double acc[F], sq[2] = {0.0, 0.0};
#pragma unroll
    for (int f = 0; f < F; ++f) acc[f] = 0.0;
    auto add_row = [&](int32_t m) {
        const T *row = Xb + (size_t)pb[m] * D + sub * F;
#pragma unroll
        for (int v = 0; v < F / VEC; ++v) {
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(row) + v);
            const T *e = reinterpret_cast<const T *>(&u);
#pragma unroll
            for (int i = 0; i < VEC; ++i) {
                const double x = (double)to_float(e[i]);
                const int f = v * VEC + i;
                acc[f] += x;
                sq[f & 1] = fma(x, x, sq[f & 1]);
            }
        }
    };
    int32_t m = s0 + grp;
    for (; m + 12 < s1; m += 16) {   // four members of this group per iteration, in order
        add_row(m);
        add_row(m + 4);
        add_row(m + 8);
        add_row(m + 12);
    }
    for (; m < s1; m += 4) add_row(m);
    // combine the 4 groups in order: (g0 + g1) + (g2 + g3)
#pragma unroll
    for (int f = 0; f < F; ++f) {
        const double o8 = __shfl_xor_sync(0xffffffffu, acc[f], 8);
        const double a01 = (grp & 1) ? o8 + acc[f] : acc[f] + o8;
        const double o16 = __shfl_xor_sync(0xffffffffu, a01, 16);
        acc[f] = (grp & 2) ? o16 + a01 : a01 + o16;
    }
    double dist = sq[0] + sq[1];
    {
        const double o8 = __shfl_xor_sync(0xffffffffu, dist, 8);
        const double a01 = (grp & 1) ? o8 + dist : dist + o8;
        const double o16 = __shfl_xor_sync(0xffffffffu, a01, 16);
        dist = (grp & 2) ? o16 + a01 : a01 + o16;
    }
    {   // sum over the members of |x - c|^2 for this lane's features
        double cx = 0.0, cc = 0.0;
#pragma unroll
        for (int f = 0; f < F; ++f) {
            const double c = (double)cr[f];
            cx = fma(c, acc[f], cx);
            cc = fma(c, c, cc);
        }
        dist = dist - 2.0 * cx + (double)cnt * cc;
    }
    if (grp == 0) {
        float *out = newC + ((size_t)b * K + k) * D + sub * F;
#pragma unroll
        for (int f = 0; f < F; ++f) out[f] = cnt > 0 ? (float)(acc[f] / (double)cnt) : cr[f];
    }
#pragma unroll
    for (int o = 4; o; o >>= 1) dist += __shfl_xor_sync(0xffffffffu, dist, o);
    if (lane == 0) segin[seg] = dist;
}

// Inertia: per problem (one block each), the segments' fp64 distance sums:
// thread t adds clusters t, t + 256, ... in order, then a fixed tree.
__global__ void __launch_bounds__(256) km_inertia_kernel(const double *__restrict__ segin, int K,
                                                         double *__restrict__ inertia) {
    __shared__ double part[256];
    const int b = blockIdx.x, t = threadIdx.x;
    double s = 0.0;
    for (int k = t; k < K; k += 256) s += segin[(size_t)b * K + k];
    part[t] = s;
    __syncthreads();
    for (int o = 128; o; o >>= 1) {
        if (t < o) part[t] += part[t + o];
        __syncthreads();
    }
    if (t == 0) inertia[b] = part[0];
}

template <typename T>
static cudaError_t launch_kmeans_t(const T *X, int B, int64_t N, int d, int K, const float *C,
                                   int32_t *ids, float *newC, int32_t *counts, double *inertia,
                                   char *ws, const KmWsLayout &L, uint32_t flags,
                                   cudaStream_t s) {
    float *mind = (float *)(ws + L.off_mind);
    int32_t *hist = (int32_t *)(ws + L.off_hist);
    int32_t *perm = (int32_t *)(ws + L.off_perm);
    int32_t *segoff = (int32_t *)(ws + L.off_segoff);
    double *inpart = (double *)(ws + L.off_inpart);
    bool tc_done = false;
    if (!(flags & GMM_FLAG_FORCE_SIMT)) {
        const gmm_dtype dt = std::is_same<T, float>::value  ? GMM_F32
                             : std::is_same<T, __half>::value ? GMM_F16
                                                              : GMM_BF16;
        cudaError_t e = launch_km_tc_assign((const void *)X, dt, B, N, d, K, C, ids,
                                            ws + L.off_cnorm, (int *)ws, &tc_done, s);
        if (e != cudaSuccess) return e;
    }
    if (!tc_done) {
        const int used_tiles = (int)((N + kKmTileP - 1) / kKmTileP);
        dim3 g1(used_tiles, B);
        timer_begin(s);
        km_simt_assign_kernel<T><<<g1, 256, 0, s>>>(X, N, d, K, C, ids, mind, inpart,
                                                    L.assign_tiles);
        timer_end(s);
        note_launches(1);
    }
    dim3 g2(L.nblk, B);
    km_hist_kernel<<<g2, 256, K * sizeof(int32_t), s>>>(ids, N, K, L.nblk, hist);
    // 32-bit indices while every index the kernel forms (up to E plus a
    // batch of rounds past a warp's range) stays far below 2^31
    if ((int64_t)K * L.nblk < ((int64_t)1 << 30))
        km_scan_kernel<int32_t><<<B, 1024, 0, s>>>(hist, N, K, L.nblk, segoff);
    else
        km_scan_kernel<int64_t><<<B, 1024, 0, s>>>(hist, N, K, L.nblk, segoff);
    size_t sc_smem = 8 * (size_t)K * sizeof(int32_t);
    cudaError_t e = cudaFuncSetAttribute(km_scatter_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sc_smem);
    if (e != cudaSuccess) return e;
    km_scatter_kernel<<<g2, 256, sc_smem, s>>>(ids, N, K, L.nblk, hist, perm);
    int64_t segs = (int64_t)B * K;
    double *segin = (double *)(ws + L.off_segin);
    const unsigned sgrid = (unsigned)((segs * 32 + 255) / 256);
    if (d == 128)
        km_segreduce_vec_kernel<T, 128><<<sgrid, 256, 0, s>>>(X, B, N, K, perm, segoff, C, newC,
                                                              counts, segin);
    else if (d == 64)
        km_segreduce_vec_kernel<T, 64><<<sgrid, 256, 0, s>>>(X, B, N, K, perm, segoff, C, newC,
                                                             counts, segin);
    else
        km_segreduce_kernel<T><<<sgrid, 256, 0, s>>>(X, B, N, d, K, perm, segoff, C, newC, counts,
                                                     segin);
    if (inertia) km_inertia_kernel<<<B, 256, 0, s>>>(segin, K, inertia);
    note_launches(4 + (inertia ? 1 : 0));
    return cudaGetLastError();
}

// Member variances of each cluster of the last partition (one warp per
// cluster, lanes over features, members in segment order, fp64 sums of
// (x - mean)^2): the hard-assignment M-step's variance.
template <typename T>
__global__ void __launch_bounds__(256)
km_member_vars_kernel(const T *__restrict__ X, int d, int K, const int32_t *__restrict__ perm,
                      const int32_t *__restrict__ segoff, const float *__restrict__ means,
                      float var_floor, float *__restrict__ vars) {
    const int k = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    if (k >= K) return;
    const int32_t s0 = segoff[k], s1 = segoff[k + 1];
    for (int j = lane; j < d; j += 32) {
        const double c = (double)means[(size_t)k * d + j];
        double acc = 0.0;
        for (int32_t m = s0; m < s1; ++m) {
            const double x = (double)load_elem<T>(X + (size_t)perm[m] * d + j);
            acc += (x - c) * (x - c);
        }
        double v = s1 > s0 ? acc / (double)(s1 - s0) : 1.0;
        if (v < (double)var_floor) v = (double)var_floor;
        vars[(size_t)k * d + j] = (float)v;
    }
}

cudaError_t launch_km_member_vars(const void *X, gmm_dtype dt, int64_t N, int d, int K,
                                  const void *ws, const float *means, float var_floor,
                                  float *vars, cudaStream_t s) {
    const KmWsLayout L = km_ws_layout(1, N, d, K);
    const char *w = (const char *)ws;
    const int32_t *perm = (const int32_t *)(w + L.off_perm);
    const int32_t *segoff = (const int32_t *)(w + L.off_segoff);
    const unsigned grid = (unsigned)(((int64_t)K * 32 + 255) / 256);
    switch (dt) {
        case GMM_F32:
            km_member_vars_kernel<float><<<grid, 256, 0, s>>>((const float *)X, d, K, perm, segoff,
                                                             means, var_floor, vars);
            break;
        case GMM_BF16:
            km_member_vars_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
                (const __nv_bfloat16 *)X, d, K, perm, segoff, means, var_floor, vars);
            break;
        default:
            km_member_vars_kernel<__half><<<grid, 256, 0, s>>>((const __half *)X, d, K, perm,
                                                              segoff, means, var_floor, vars);
    }
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_kmeans(const void *X, gmm_dtype dt, int B, int64_t N, int d, int K,
                          const float *C, int32_t *ids, float *newC, int32_t *counts,
                          double *inertia, void *ws, const KmWsLayout &L, uint32_t flags,
                          cudaStream_t s) {
    char *w = (char *)ws;
    switch (dt) {
        case GMM_F32:
            return launch_kmeans_t<float>((const float *)X, B, N, d, K, C, ids, newC, counts,
                                          inertia, w, L, flags, s);
        case GMM_BF16:
            return launch_kmeans_t<__nv_bfloat16>((const __nv_bfloat16 *)X, B, N, d, K, C, ids,
                                                  newC, counts, inertia, w, L, flags, s);
        case GMM_F16:
            return launch_kmeans_t<__half>((const __half *)X, B, N, d, K, C, ids, newC, counts,
                                           inertia, w, L, flags, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace gmmb
