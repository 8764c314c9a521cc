// Tensor-core (tcgen05 / TMEM) assignment step of Lloyd k-means.
//
// What is computed ("Flash-KMeans gor k-means realtime-venligt pa GPU ...",
// section "FlashAssign gor tildelingen hurtig": point and centroid tiles are
// streamed through on-chip memory and only a running (best distance, best
// index) per point is kept): for each point x_n of problem b,
//     id_n = argmin_k  D'_nk,   D'_nk = ||c_k||^2 - 2 x_n . c_k
// (the squared distance minus ||x_n||^2, which does not depend on k), ties to
// the lowest k.  The contraction x . c runs on the tensor core, 128 points x
// 256 centroids per MMA tile, accumulated in TMEM; the N x K matrix is never
// written.
//
// Precision: kind::f16 (fp16 x fp16 -> fp32).  Centroids are split into fp16
// pieces c = c_hi + c_lo (about 22 significant bits), points likewise when
// they are fp32 (16-bit points are exact in fp16), and a product is
// x_hi c_hi + x_hi c_lo (+ x_lo c_hi), small terms first.  The argmin is then
// exact except where two distances differ by about 2^-21 of ||x||^2 + ||c||^2.
//
// Warp roles (320 threads): warp 0 streams centroid piece stages (1-D bulk
// copies into a ring), warp 1 issues tcgen05.mma, warps 2-9 convert point
// tiles into fp16 pieces and read TMEM (running argmin per point; warps 2-5
// take the first 128 centroids of each chunk, 6-9 the second 128).  Every wait
// is bounded (tc::mbar_wait).
#include "common.cuh"
#include "kmeans_tc.h"
#include "tc_ptx.cuh"

#include <math.h>
#include <type_traits>

namespace gmmb {
using namespace tc;

namespace {

constexpr int kKtTile = 128;               // points per tile = MMA M
constexpr int kKtChunk = 256;              // centroids per chunk = MMA N
constexpr int kKtThreads = 320;
constexpr int kKtBlock = kKtTile * 128;    // one 64-feature block of a 128-row tile (16 KB)
constexpr int kKtStage = kKtChunk * 128;   // one 64-feature block of a 256-row chunk (32 KB)
constexpr int kKtStages = 4;
constexpr float kKtRange = 65504.f;        // fp16 max

int kt_kp(int K) { return (K + kKtChunk - 1) / kKtChunk * kKtChunk; }

// Centroid image per problem: [piece (0 hi, 1 lo)][64-feature block][Kp rows][128 B],
// SWIZZLE_128B K-major; padded rows are zero and get ||c||^2 = +inf.
__host__ __device__ inline size_t kt_img_bytes(int Kp, int NB) { return (size_t)2 * NB * Kp * 128; }

template <int NB, bool XSPLIT>
struct KtSmem {
    static constexpr int XPIECES = XSPLIT ? 2 : 1;     // x_hi [, x_lo]
    static constexpr int XP = XPIECES * NB * kKtBlock;
    static constexpr int RING = XP;
    static constexpr int XCH = RING + kKtStages * kKtStage;   // (best, idx) of the second half
    static constexpr int BARS = XCH + kKtTile * 8;
    static constexpr int MISC = BARS + 256;
    static constexpr int TOTAL = MISC + 256 + 1024;          // + alignment slack
    static_assert(TOTAL <= 232448, "shared memory budget");
};

struct KtBars {
    uint64_t wfull[kKtStages], wempty[kKtStages];
    uint64_t xfull, xfree;
    uint64_t sfull[2], sfree[2];
    uint64_t rsync;
    uint64_t done;
};

template <typename XT>
__device__ __forceinline__ void kt_load8(const XT *p, float (&v)[8]);
template <>
__device__ __forceinline__ void kt_load8<float>(const float *p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
    const float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
__device__ __forceinline__ void kt_load8<__half>(const __half *p, float (&v)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) { const float2 f = __half22float2(h[i]); v[2 * i] = f.x; v[2 * i + 1] = f.y; }
}
template <>
__device__ __forceinline__ void kt_load8<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

__device__ __forceinline__ uint32_t kt_h2u(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }

}  // namespace

// Centroid pieces and norms.  One warp per (problem, padded centroid row).
__global__ void km_tc_params_kernel(const float *__restrict__ C, int B, int K, int d, int Kp,
                                    uint8_t *__restrict__ img, float *__restrict__ cn, int *err) {
    const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= (int64_t)B * Kp) return;
    const int b = (int)(warp / Kp), k = (int)(warp % Kp);
    const int NB = d / 64;
    uint8_t *ib = img + (size_t)b * kt_img_bytes(Kp, NB);
    double nrm = 0.0;
    bool bad = false;
    for (int j = lane; j < d; j += 32) {
        const float c = k < K ? C[((size_t)b * K + k) * d + j] : 0.f;
        bad |= !(fabsf(c) < kKtRange);
        nrm += (double)c * (double)c;
        const __half hi = __float2half_rn(c);
        const __half lo = __float2half_rn(c - __half2float(hi));
        const int blk = j / 64, f = j % 64;
        const size_t off = swz128_off((uint32_t)k, (uint32_t)f >> 3) + (f & 7) * 2;
        *reinterpret_cast<__half *>(ib + ((size_t)(0 * NB + blk) * Kp) * 128 + off) = hi;
        *reinterpret_cast<__half *>(ib + ((size_t)(1 * NB + blk) * Kp) * 128 + off) = lo;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) nrm += __shfl_xor_sync(0xffffffffu, nrm, o);
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_error(err, GMM_ERR_RANGE);
    if (lane == 0) cn[(size_t)b * Kp + k] = k < K ? (float)nrm : INFINITY;
}

template <int NB, typename XT>
__global__ void __launch_bounds__(kKtThreads, 1)
km_tc_assign_kernel(const XT *__restrict__ X, int B, int64_t N, int Kp,
                    const uint8_t *__restrict__ img, const float *__restrict__ cn,
                    int32_t *__restrict__ ids, int *err) {
    constexpr bool XSPLIT = std::is_same<XT, float>::value;
    using S = KtSmem<NB, XSPLIT>;
    constexpr int D = NB * 64;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    KtBars *bars = reinterpret_cast<KtBars *>(sm + S::BARS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S::MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + S::MISC + 4);
    float2 *xch = reinterpret_cast<float2 *>(sm + S::XCH);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t T = (N + kKtTile - 1) / kKtTile;   // tiles per problem
    const int64_t items = (int64_t)B * T;
    const int nchunks = Kp / kKtChunk;
    constexpr int kStages = 2 * NB;                  // per chunk: (c_lo, c_hi) per block
    const size_t img_per_b = kt_img_bytes(Kp, NB);

    if (tid == 0) {
        for (int s = 0; s < kKtStages; ++s) { mbar_init(&bars->wfull[s], 1); mbar_init(&bars->wempty[s], 1); }
        mbar_init(&bars->xfull, 8);
        mbar_init(&bars->xfree, 1);
        for (int b = 0; b < 2; ++b) { mbar_init(&bars->sfull[b], 1); mbar_init(&bars->sfree[b], 8); }
        mbar_init(&bars->rsync, 8);
        mbar_init(&bars->done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;   // two score buffers of 256 columns

    if (warp == 0) {
        // ===================== centroid-piece producer
        if (lane == 0) {
            uint32_t g = 0;
            for (int64_t item = blockIdx.x; item < items && !*abort_flag; item += gridDim.x) {
                const uint8_t *ib = img + (size_t)(item / T) * img_per_b;
                for (int c = 0; c < nchunks && !*abort_flag; ++c) {
                    for (int i = 0; i < kStages; ++i, ++g) {
                        const int blk = i >> 1, piece = (i & 1) ? 0 : 1;   // c_lo first, then c_hi
                        const int slot = g % kKtStages;
                        if (!mbar_wait(&bars->wempty[slot], ((g / kKtStages) & 1) ^ 1, err, abort_flag))
                            goto producer_done;
                        mbar_arrive_expect_tx(&bars->wfull[slot], kKtStage);
                        bulk_g2s(sm + S::RING + slot * kKtStage,
                                 ib + ((size_t)(piece * NB + blk) * Kp + (size_t)c * kKtChunk) * 128,
                                 kKtStage, &bars->wfull[slot]);
                    }
                }
            }
        producer_done:
            for (uint32_t i = 0; i < (uint32_t)kKtStages && i < g; ++i) {
                const uint32_t gg = g - 1 - i;
                mbar_wait_drain(&bars->wfull[gg % kKtStages], (gg / kKtStages) & 1, err);
            }
        }
    } else if (warp == 1) {
        // ===================== MMA issuer.  The descriptors are built once and
        // the chunk's stage program is unrolled, so each MMA costs the issuing
        // thread two adds (its issue rate bounds the tensor core otherwise).
        if (lane == 0) {
            const uint32_t idesc = idesc_f16(kKtTile, kKtChunk, false, false);
            const uint64_t dX = smem_desc(smem_u32(sm), 16, 1024, kSwz128);
            const uint64_t dR = smem_desc(smem_u32(sm + S::RING), 16, 1024, kSwz128);
            uint32_t slot = 0, sph = 0, q = 0;
            int it = 0;
            bool ok = true;
            for (int64_t item = blockIdx.x; item < items && ok; item += gridDim.x, ++it) {
                if (!mbar_wait(&bars->xfull, it & 1, err, abort_flag)) { ok = false; break; }
                for (int c = 0; c < nchunks && ok; ++c, ++q) {
                    const uint32_t buf = q & 1;
                    if (!mbar_wait(&bars->sfree[buf], ((q >> 1) & 1) ^ 1, err, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t dS = tmem + buf * kKtChunk;
#pragma unroll
                    for (int i = 0; i < kStages; ++i) {
                        const int blk = i >> 1;
                        const bool lo = !(i & 1);
                        if (!mbar_wait(&bars->wfull[slot], sph, err, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        const uint64_t db = dR + slot * (uint32_t)(kKtStage >> 4);
                        const uint64_t dxh = dX + (uint32_t)(((0 * NB + blk) * kKtBlock) >> 4);
                        const uint64_t dxl = dX + (uint32_t)(((1 * NB + blk) * kKtBlock) >> 4);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            if (lo) {
                                mma_f16(dS, dxh + 2 * kk, db + 2 * kk, idesc, (i | kk) ? 1u : 0u);
                            } else {
                                if (XSPLIT) mma_f16(dS, dxl + 2 * kk, db + 2 * kk, idesc, 1u);
                                mma_f16(dS, dxh + 2 * kk, db + 2 * kk, idesc, 1u);
                            }
                        }
                        mma_commit(&bars->wempty[slot]);
                        if (++slot == kKtStages) { slot = 0; sph ^= 1; }
                    }
                    if (!ok) break;
                    mma_commit(&bars->sfull[buf]);
                    if (c == nchunks - 1) mma_commit(&bars->xfree);
                }
            }
            mma_commit(&bars->done);
            mbar_wait_drain(&bars->done, 0, err);   // no MMA in flight at teardown
        }
    } else {
        // ===================== workers: point-tile conversion and the running argmin
        const int qd = warp & 3;                   // TMEM lane quadrant
        const int h = (warp - 2) >> 2;             // centroid half of each chunk
        const int p = qd * 32 + lane;              // TMEM lane = point row
        const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
        uint32_t q = 0, rs = 0;
        auto reader_sync = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->rsync);
            const bool r = mbar_wait(&bars->rsync, rs & 1, err, abort_flag);
            ++rs;
            return r;
        };
        const int ct = tid - 64;
        constexpr int CPR = D / 8;                 // 16-byte chunks per row
        constexpr int GROUPS = kKtTile * CPR / 256;
        auto convert_tile = [&](int64_t item, int it) -> bool {
            const int64_t b = item / T, t = item % T;
            const XT *Xb = X + (size_t)b * N * D;
            float v[GROUPS][8];
#pragma unroll
            for (int i = 0; i < GROUPS; ++i) {
                const int gi = ct + 256 * i;
                const int pr = gi / CPR, c = gi % CPR;
                const int64_t n = t * kKtTile + pr;
                if (n < N) {
                    kt_load8<XT>(Xb + n * D + c * 8, v[i]);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[i][e] = 0.f;
                }
            }
            if (it > 0 && !mbar_wait(&bars->xfree, (it - 1) & 1, err, abort_flag)) return false;
            bool bad = false;
#pragma unroll
            for (int i = 0; i < GROUPS; ++i) {
                const int gi = ct + 256 * i;
                const int pr = gi / CPR, c = gi % CPR;
                const int blk = c / 8;
                const uint32_t off = swz128_off(pr, c % 8);
                uint32_t wh[4], wl[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const float x0 = v[i][e], x1 = v[i][e + 1];
                    bad |= !(fabsf(x0) < kKtRange) || !(fabsf(x1) < kKtRange);
                    const __half2 hh = __floats2half2_rn(x0, x1);
                    wh[e / 2] = kt_h2u(hh);
                    if (XSPLIT) {
                        const float2 hf = __half22float2(hh);
                        wl[e / 2] = kt_h2u(__floats2half2_rn(x0 - hf.x, x1 - hf.y));
                    }
                }
                *reinterpret_cast<uint4 *>(sm + (0 * NB + blk) * kKtBlock + off) =
                    make_uint4(wh[0], wh[1], wh[2], wh[3]);
                if (XSPLIT)
                    *reinterpret_cast<uint4 *>(sm + (1 * NB + blk) * kKtBlock + off) =
                        make_uint4(wl[0], wl[1], wl[2], wl[3]);
            }
            if (__any_sync(0xffffffffu, bad) && lane == 0) set_error(err, GMM_ERR_RANGE);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->xfull);
            return true;
        };

        int it = 0;
        bool live = (int64_t)blockIdx.x >= items || convert_tile(blockIdx.x, 0);
        // the next tile is converted before the last two chunks are read (its
        // X pieces are released after the last chunk's MMAs, which wait for the
        // reading of the chunk two back)
        const int conv_at = nchunks >= 2 ? nchunks - 2 : 0;
        for (int64_t item = blockIdx.x; item < items && live; item += gridDim.x, ++it) {
            const int64_t b = item / T, t = item % T;
            const int64_t n = t * kKtTile + p;
            const bool has_next = item + gridDim.x < items;
            const float *cnb = cn + (size_t)b * Kp;
            float best = INFINITY;
            int bidx = 0x7fffffff;
            bool ok = true;
            for (int c = 0; c < nchunks; ++c, ++q) {
                if (c == conv_at && has_next && !convert_tile(item + gridDim.x, it + 1)) { ok = false; break; }
                const uint32_t buf = q & 1;
                if (!mbar_wait(&bars->sfull[buf], (q >> 1) & 1, err, abort_flag)) { ok = false; break; }
                tc_fence_after();
#pragma unroll 1
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t r[32];
                    const int col = h * 128 + cc * 32;
                    const int kb = c * kKtChunk + col;
                    tmem_ld32(tmem + lane_base + buf * kKtChunk + col, r);
                    float dv[32];
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        const float4 nv = __ldg(reinterpret_cast<const float4 *>(cnb + kb + i));
                        dv[i] = nv.x; dv[i + 1] = nv.y; dv[i + 2] = nv.z; dv[i + 3] = nv.w;
                    }
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) dv[i] = fmaf(-2.f, __uint_as_float(r[i]), dv[i]);
                    // argmin of the 32 as a tree (the lower index of a pair is
                    // kept unless the higher one is strictly smaller), then one
                    // strict comparison with the running best: ties go to the
                    // lowest index either way
                    int iv[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) iv[i] = i;
#pragma unroll
                    for (int n = 16; n >= 1; n >>= 1) {
#pragma unroll
                        for (int j = 0; j < n; ++j) {
                            const bool up = dv[2 * j + 1] < dv[2 * j];
                            dv[j] = up ? dv[2 * j + 1] : dv[2 * j];
                            iv[j] = up ? iv[2 * j + 1] : iv[2 * j];
                        }
                    }
                    if (dv[0] < best) { best = dv[0]; bidx = kb + iv[0]; }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->sfree[buf]);
            }
            if (!ok) break;
            // merge the two centroid halves: smaller distance, then smaller index
            if (h == 1) xch[p] = make_float2(best, __int_as_float(bidx));
            if (!reader_sync()) break;
            if (h == 0 && n < N) {
                const float ob = xch[p].x;
                const int oi = __float_as_int(xch[p].y);
                if (ob < best || (ob == best && oi < bidx)) bidx = oi;
                ids[(size_t)b * N + n] = bidx;
            }
            if (!reader_sync()) break;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- host side

int km_tc_tiles_per_problem(int64_t N) { return (int)((N + kKtTile - 1) / kKtTile); }

size_t km_tc_param_bytes(int B, int d, int K) {
    if (d != 64 && d != 128) return 0;
    const int Kp = kt_kp(K);
    return align_up((size_t)B * kt_img_bytes(Kp, d / 64)) + align_up((size_t)B * Kp * 4);
}

static int kt_sm_count() {
    static int cached = 0;
    if (!cached) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&cached, cudaDevAttrMultiProcessorCount, dev);
        if (cached <= 0) cached = 148;
    }
    return cached;
}

template <int NB, typename XT>
static cudaError_t kt_launch(const XT *X, int B, int64_t N, int Kp, const uint8_t *img,
                             const float *cn, int32_t *ids, int *err, cudaStream_t s) {
    auto kern = km_tc_assign_kernel<NB, XT>;
    const int smem = KtSmem<NB, std::is_same<XT, float>::value>::TOTAL;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int64_t items = (int64_t)B * ((N + kKtTile - 1) / kKtTile);
    int grid = kt_sm_count();
    if (grid > items) grid = (int)items;
    kern<<<grid, kKtThreads, smem, s>>>(X, B, N, Kp, img, cn, ids, err);
    return cudaGetLastError();
}

cudaError_t launch_km_tc_assign(const void *X, gmm_dtype dt, int B, int64_t N, int d, int K,
                                const float *C, int32_t *ids, void *param_ws, int *err,
                                bool *done, cudaStream_t s) {
    *done = false;
    if (d != 64 && d != 128) return cudaSuccess;   // the CUDA-core kernel takes it
    const int Kp = kt_kp(K), NB = d / 64;
    uint8_t *img = (uint8_t *)param_ws;
    float *cn = (float *)((char *)param_ws + align_up((size_t)B * kt_img_bytes(Kp, NB)));
    const int64_t rows = (int64_t)B * Kp;
    km_tc_params_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, s>>>(C, B, K, d, Kp, img,
                                                                            cn, err);
    note_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    timer_begin(s);
    if (NB == 2) {
        if (dt == GMM_F32) e = kt_launch<2, float>((const float *)X, B, N, Kp, img, cn, ids, err, s);
        else if (dt == GMM_BF16)
            e = kt_launch<2, __nv_bfloat16>((const __nv_bfloat16 *)X, B, N, Kp, img, cn, ids, err, s);
        else e = kt_launch<2, __half>((const __half *)X, B, N, Kp, img, cn, ids, err, s);
    } else {
        if (dt == GMM_F32) e = kt_launch<1, float>((const float *)X, B, N, Kp, img, cn, ids, err, s);
        else if (dt == GMM_BF16)
            e = kt_launch<1, __nv_bfloat16>((const __nv_bfloat16 *)X, B, N, Kp, img, cn, ids, err, s);
        else e = kt_launch<1, __half>((const __half *)X, B, N, Kp, img, cn, ids, err, s);
    }
    timer_end(s);
    note_launches(1);
    if (e == cudaSuccess) *done = true;
    return e;
}

}  // namespace gmmb
