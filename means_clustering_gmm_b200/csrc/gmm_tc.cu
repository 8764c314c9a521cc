// Tensor-core (tcgen05 / TMEM) fused GMM E-step for sm_100a.
//
// What is computed (see "Turbo-GMM: FlashAttention-Inspired GPU-Accelerated
// Gaussian Mixture Model", abstract, and "Flash-GMM: a memory-efficient kernel
// for scalable soft clustering", abstract): the scores of a 128-point tile
// against the components are a dense contraction on the tensor core,
//     s_nk = 2^e_k * ( sum_j x_nj W1'_kj + sum_j x_nj^2 W2'_kj ) + c_k,
//     W1 = mu / var, W2 = -1 / (2 var), c_k = log w_k - 1/2 sum_j (mu^2/var + log 2 pi var),
// (W' = W * 2^-e_k, a per-component power of two that keeps the fp16 pieces
// in range), held in TMEM and never written to memory; the responsibilities
// r_nk = exp(s_nk - l_n) go to shared memory, and a second tcgen05
// contraction R^T [X, X o X] accumulates the sufficient statistics in TMEM
// across all tiles of the CTA.
//
// Regimes ("Turbo-GMM", abstract: single sweep when the component axis fits on
// chip, otherwise the two-pass design that recomputes the scores):
//   single sweep (K <= 128):  one kernel; the whole score row is in TMEM.
//   two sweeps   (K  > 128):  sweep 1 (kMode = kLse) computes l_n with an
//                              online max/sum over 256-component chunks;
//                              sweep 2 (kMode = kStats) recomputes the scores
//                              of one 128-component slice per CTA and
//                              accumulates that slice's statistics.
//
// Precision: the MMA kind is f16 (fp16 x fp16 -> fp32).  Every fp32 operand
// is split into an fp16 pair hi + lo (22 significant bits) and products
// hi*hi + hi*lo + lo*hi are accumulated, so the contraction carries ~2^-21
// relative error per term instead of fp16's 2^-11:
//   E-step  A = [x_hi, x_lo, x^2_hi, x^2_lo] (K-major, 128 points),
//           B = [W1_hi, W1_lo, W2_hi, W2_lo] (K-major, components),
//   M-step  A = [r_hi, r_lo]^T (MN-major: components contiguous),
//           B = [x_hi | x^2_hi], [x_lo | x^2_lo] (MN-major: the same X tile).
// 16-bit inputs are exact in fp16 (x_lo = 0), so their x_lo products are
// skipped.  |x| must be below 181 (x^2 within fp16); the converter flags
// GMM_ERR_RANGE otherwise.
//
// Warp roles (512 threads): warp 0 streams the parameter pieces (1-D bulk
// copies into a ring), warp 1 issues tcgen05.mma, warps 4-7 read TMEM
// (scores, then the statistics), warps 8-15 convert X tiles into the fp16
// pieces.  All waits are bounded (tc::mbar_wait).
#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

#include <math.h>
#include <type_traits>

namespace gmmb {
using namespace tc;

namespace {

constexpr int kTileP = 128;     // points per tile = MMA M of the E-step
constexpr int kSlice = 128;     // components per CTA in sweep 2 / single sweep
constexpr int kChunk1 = 256;    // components per chunk in sweep 1
constexpr int kThreads = 512;
constexpr int kBlockBytes = kTileP * 128;  // one 64-feature block of a 128-row tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRangeMax = 181.0f;        // 181^2 < 65504 (fp16 max)
// Initial responsibility scale exponent: r < 2^-100 never matters (such a
// component has N_k < 1e-12 N for any N below 2^60 and is kept as it was).
constexpr int kSigInit = 115;

enum Mode { kLse = 0, kStats = 1, kSingle = 2 };

// Parameter image in global memory, fp16, laid out so that any 128- or
// 256-component chunk of one (piece, feature block) is one contiguous run of
// 128-byte rows in the SWIZZLE_128B K-major order the MMA reads:
//   image[piece][block][Kp rows][128 B],  piece: 0 W1_hi, 1 W1_lo, 2 W2_hi, 3 W2_lo.
// Padded components (k >= K) have zero pieces, a_k = 0 and b_k = -inf.
struct TcParams {
    const uint8_t *img;
    const float *ak;   // 2^e_k * log2(e)
    const float *bk;   // c_k * log2(e)
    int Kp;
};

__host__ __device__ inline size_t img_bytes(int Kp, int NB) {
    return (size_t)4 * NB * Kp * 128;
}
__host__ __device__ inline size_t img_off(int piece, int block, int k, int NB, int Kp) {
    return (((size_t)piece * NB + block) * Kp + k) * 128;
}
// byte offset of element (component k, feature f of block `block`) of a piece
__host__ __device__ inline size_t img_elem(int piece, int block, int k, int f, int NB, int Kp) {
    return img_off(piece, block, 0, NB, Kp) + (size_t)(k >> 3) * 1024 +
           swz128_off(k & 7, f >> 3) + (f & 7) * 2;
}

}  // namespace

// a1: W pieces, per-component scale and constant.  One warp per component.
__global__ void gmm_tc_params_kernel(const float *__restrict__ means,
                                     const float *__restrict__ vars,
                                     const float *__restrict__ logw, int K, int d, int Kp,
                                     uint8_t *__restrict__ img, float *__restrict__ ak,
                                     float *__restrict__ bk, int *err) {
    const int warp = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    if (warp >= Kp) return;
    const int k = warp;
    const int NB = d / 64;
    if (k >= K) {
        for (int j = lane; j < d; j += 32)
            for (int pc = 0; pc < 4; ++pc)
                *reinterpret_cast<__half *>(img + img_elem(pc, j / 64, k, j % 64, NB, Kp)) =
                    __float2half_rn(0.f);
        if (lane == 0) { ak[k] = 0.f; bk[k] = -INFINITY; }
        return;
    }
    // max |W| for the scale, and the constant in fp64 (fixed butterfly order)
    double mx = 0.0, cacc = 0.0;
    for (int j = lane; j < d; j += 32) {
        double mu = means[(size_t)k * d + j], v = vars[(size_t)k * d + j];
        double w1 = mu / v, w2 = -0.5 / v;
        mx = fmax(mx, fmax(fabs(w1), fabs(w2)));
        cacc += mu * mu / v + log(2.0 * M_PI * v);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        cacc += __shfl_xor_sync(0xffffffffu, cacc, o);
    }
    int ex = 0;
    frexp(mx, &ex);          // mx < 2^ex
    const int e = ex - 8;    // |W| * 2^-e < 2^8
    const double inv = ldexp(1.0, -e);
    if (!(mx > 0.0) || !isfinite(mx)) set_error(err, GMM_ERR_RANGE);
    for (int j = lane; j < d; j += 32) {
        double mu = means[(size_t)k * d + j], v = vars[(size_t)k * d + j];
        double w[2] = {mu / v * inv, -0.5 / v * inv};
        for (int t = 0; t < 2; ++t) {
            __half hi = __float2half_rn((float)w[t]);
            __half lo = __float2half_rn((float)(w[t] - (double)__half2float(hi)));
            *reinterpret_cast<__half *>(img + img_elem(2 * t, j / 64, k, j % 64, NB, Kp)) = hi;
            *reinterpret_cast<__half *>(img + img_elem(2 * t + 1, j / 64, k, j % 64, NB, Kp)) = lo;
        }
    }
    if (lane == 0) {
        double c = (double)logw[k] - 0.5 * cacc;
        ak[k] = (float)(ldexp(1.0, e) * (double)kLog2e);
        bk[k] = (float)(c * (double)kLog2e);
    }
}

namespace {

// Shared-memory plan of the fused kernel (bytes, offsets from a 1024-aligned base).
template <int NB, int MODE>
struct Smem {
    static constexpr int C = (MODE == kLse) ? kChunk1 : kSlice;   // components per chunk
    static constexpr int XP = 4 * NB * kBlockBytes;               // X pieces
    static constexpr int STAGE = C * 128;                         // one W stage
    static constexpr int NSTAGE = (MODE == kLse) ? 3 : 5;
    static constexpr int RING = XP;                               // ring offset
    static constexpr int RBYTES = 2 * 2 * kBlockBytes;            // r_hi, r_lo (2 comp blocks)
    static constexpr int ONES = RING + NSTAGE * STAGE;            // 16 x 128 fp16 ones
    static constexpr int ONES_BYTES = (MODE == kLse) ? 0 : 4096;
    static constexpr int CONSTS = ONES + ONES_BYTES;              // a_k, b_k of the slice
    // a_k, b_k (2 x 128 fp32), per-warp tile maxima (4 x 128 int), scales (128 int)
    static constexpr int CONSTS_BYTES = (MODE == kLse) ? 0 : 7 * kSlice * 4;
    static constexpr int BARS = CONSTS + CONSTS_BYTES;
    static constexpr int BARS_BYTES = 256;
    static constexpr int MISC = BARS + BARS_BYTES;                // tmem addr, abort, ll scratch
    static constexpr int TOTAL = MISC + 256 + 1024;               // + alignment slack
    static_assert(MODE == kLse || RBYTES <= NSTAGE * STAGE, "R must fit in the ring");
};

// Order in which the parameter stages (one piece of one 64-feature block, for
// the chunk's components) are streamed and consumed by the E-step:
//   phase 1, per block: W1_lo (x x_hi), W2_lo (x x2_hi), [W1_hi (x x_lo),
//            fp32 inputs only], W2_hi (x x2_lo)   -- the small products
//   phase 2, per block: W1_hi and W2_hi together  -- the large products,
//            interleaved per 16-feature step.
template <int NB, bool XEXACT>
struct EProg {
    static constexpr int kP1 = XEXACT ? 3 : 4;
    static constexpr int kStages1 = NB * kP1;
    static constexpr int kStages = kStages1 + 2 * NB;
    __device__ static void stage(int i, int &pc, int &b) {
        if (i < kStages1) {
            b = i / kP1;
            const int t = i % kP1;
            pc = (t == 0) ? 1 : (t == 1) ? 3 : (XEXACT ? 2 : (t == 2 ? 0 : 2));
        } else {
            const int t = i - kStages1;
            b = t / 2;
            pc = (t % 2 == 0) ? 0 : 2;
        }
    }
};

struct Bars {
    uint64_t wfull[6], wempty[6];
    uint64_t xfull, xfree;
    uint64_t sfull[2], sfree[2];
    uint64_t rfull, done;
};

__device__ __forceinline__ uint32_t pack_half2(__half a, __half b) {
    return (uint32_t)__half_as_ushort(a) | ((uint32_t)__half_as_ushort(b) << 16);
}

template <typename XT>
__device__ __forceinline__ void load8(const XT *p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<float>(const float *p, float (&v)[8]) {
    float4 a = __ldg(reinterpret_cast<const float4 *>(p));
    float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<__half>(const __half *p, float (&v)[8]) {
    uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) { float2 f = __half22float2(h[i]); v[2 * i] = f.x; v[2 * i + 1] = f.y; }
}
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[8]) {
    uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

}  // namespace

// The fused kernel.  MODE kLse: grid = persistent CTAs over point tiles.
// MODE kStats / kSingle: grid = (component slices, point ranges).
template <int NB, typename XT, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
gmm_tc_fused_kernel(const XT *__restrict__ X, int64_t N, int K, TcParams P,
                    const float *__restrict__ lse_in, float *__restrict__ lse_out,
                    float *__restrict__ loglik, double *__restrict__ ll_part,
                    float *__restrict__ partial, int *__restrict__ partial_sig,
                    int64_t tiles_per_range, int *err) {
    using S = Smem<NB, MODE>;
    constexpr int C = S::C;
    constexpr int D = NB * 64;
    constexpr bool XEXACT = !std::is_same<XT, float>::value;
    using Prog = EProg<NB, XEXACT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    Bars *bars = reinterpret_cast<Bars *>(sm + S::BARS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S::MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + S::MISC + 4);
    float *llw = reinterpret_cast<float *>(sm + S::MISC + 16);   // 4 per-warp tile sums
    float *cA = reinterpret_cast<float *>(sm + S::CONSTS);   // slice constants (sweep 2 / single)
    float *cB = cA + kSlice;
    int *tmax = reinterpret_cast<int *>(cB + kSlice);        // [4][128]
    int *sig = tmax + 4 * kSlice;                            // [128]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t ntiles = (N + kTileP - 1) / kTileP;
    // tile range of this CTA
    int64_t t_begin, t_end, t_step;
    int comp0 = 0;
    if (MODE == kLse) {
        t_begin = blockIdx.x; t_end = ntiles; t_step = gridDim.x;
    } else {
        comp0 = blockIdx.x * kSlice;
        t_begin = (int64_t)blockIdx.y * tiles_per_range;
        t_end = min(ntiles, t_begin + tiles_per_range);
        t_step = 1;
    }
    const int nchunks = (MODE == kLse) ? P.Kp / kChunk1 : 1;

    // ---- setup
    if (tid == 0) {
        for (int s = 0; s < S::NSTAGE; ++s) { mbar_init(&bars->wfull[s], 1); mbar_init(&bars->wempty[s], 1); }
        mbar_init(&bars->xfull, 8);
        mbar_init(&bars->xfree, 1);
        for (int b = 0; b < 2; ++b) { mbar_init(&bars->sfull[b], 1); mbar_init(&bars->sfree[b], 4); }
        mbar_init(&bars->rfull, 4);
        mbar_init(&bars->done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (MODE != kLse) {
        // ones block for S0 (16 rows x 128 points, any layout: all ones)
        uint32_t *ones = reinterpret_cast<uint32_t *>(sm + S::ONES);
        for (int i = tid; i < 1024; i += kThreads) ones[i] = 0x3C003C00u;
        for (int i = tid; i < kSlice; i += kThreads) {
            cA[i] = P.ak[comp0 + i];
            cB[i] = P.bk[comp0 + i];
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // TMEM columns: scores at 0 (two buffers of C in sweep 1), S0 at 128,
    // statistics at 256 (2D columns).
    const uint32_t t_s0 = tmem + 128, t_st = tmem + 256;

    if (warp == 0) {
        // ===================== parameter-piece producer
        if (lane == 0) {
            uint32_t g = 0;
            int it = 0;
            for (int64_t t = t_begin; t < t_end && !*abort_flag; t += t_step, ++it) {
                if (MODE != kLse && it > 0) {
                    // the ring aliases R: wait until the previous tile's M-step is done
                    if (!mbar_wait(&bars->xfree, (it - 1) & 1, err, abort_flag)) break;
                }
                for (int c = 0; c < nchunks && !*abort_flag; ++c) {
                    const int k0 = (MODE == kLse) ? c * kChunk1 : comp0;
                    for (int i = 0; i < Prog::kStages; ++i, ++g) {
                        int pc, b;
                        Prog::stage(i, pc, b);
                        const int slot = g % S::NSTAGE;
                        if (!mbar_wait(&bars->wempty[slot], ((g / S::NSTAGE) & 1) ^ 1, err,
                                       abort_flag))
                            goto producer_done;
                        mbar_arrive_expect_tx(&bars->wfull[slot], S::STAGE);
                        bulk_g2s(sm + S::RING + slot * S::STAGE,
                                 P.img + img_off(pc, b, k0, NB, P.Kp), S::STAGE,
                                 &bars->wfull[slot]);
                    }
                }
            }
        producer_done:
            // no bulk copy in flight at teardown
            for (uint32_t i = 0; i < (uint32_t)S::NSTAGE && i < g; ++i) {
                const uint32_t gg = g - 1 - i;
                mbar_wait_drain(&bars->wfull[gg % S::NSTAGE], (gg / S::NSTAGE) & 1, err);
            }
        }
    } else if (warp == 1) {
        // ===================== MMA issuer
        if (lane == 0) {
            const uint32_t xp = smem_u32(sm);
            const uint32_t ring = smem_u32(sm + S::RING);
            const uint32_t idesc_e = idesc_f16(128, C, false, false);
            uint32_t g = 0, q = 0;
            int it = 0;
            bool first_m = true;
            for (int64_t t = t_begin; t < t_end; t += t_step, ++it) {
                if (!mbar_wait(&bars->xfull, it & 1, err, abort_flag)) break;
                tc_fence_after();
                bool ok = true;
                for (int c = 0; c < nchunks && ok; ++c, ++q) {
                    const uint32_t buf = (MODE == kLse) ? (q & 1) : 0;
                    // sweep 1: the readers released this score buffer; sweep 2 /
                    // single: the previous tile's M-step already waited for them
                    if (MODE == kLse &&
                        !mbar_wait(&bars->sfree[buf], ((q >> 1) & 1) ^ 1, err, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t dS = tmem + buf * C;
                    // E-step program: phase 1 adds the small correction
                    // products (one operand a lo piece) while the accumulator
                    // is still small; phase 2 adds the large x_hi*W1_hi and
                    // x2_hi*W2_hi products interleaved per 16-feature step,
                    // so few additions happen at large magnitude (the tensor
                    // core's fp32 accumulation truncates).
                    uint32_t acc = 0;
                    for (int i = 0; i < Prog::kStages1 && ok; ++i, ++g) {
                        int pc, b;
                        Prog::stage(i, pc, b);
                        const int slot = g % S::NSTAGE;
                        if (!mbar_wait(&bars->wfull[slot], (g / S::NSTAGE) & 1, err, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t wb = ring + slot * S::STAGE;
                        // W1_lo x x_hi, W2_lo x x2_hi, W1_hi x x_lo, W2_hi x x2_lo
                        const int pa = (pc == 1) ? 0 : (pc == 3) ? 1 : (pc == 0) ? 2 : 3;
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint32_t a = xp + (pa * NB + b) * kBlockBytes + kk * 32;
                            mma_f16(dS, smem_desc(a, 16, 1024, kSwz128),
                                    smem_desc(wb + kk * 32, 16, 1024, kSwz128), idesc_e, acc);
                            acc = 1;
                        }
                        mma_commit(&bars->wempty[slot]);
                    }
                    for (int b = 0; b < NB && ok; ++b, g += 2) {
                        const int s1 = g % S::NSTAGE, s2 = (g + 1) % S::NSTAGE;
                        if (!mbar_wait(&bars->wfull[s1], (g / S::NSTAGE) & 1, err, abort_flag) ||
                            !mbar_wait(&bars->wfull[s2], ((g + 1) / S::NSTAGE) & 1, err, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t w1 = ring + s1 * S::STAGE, w2 = ring + s2 * S::STAGE;
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint32_t ax = xp + (0 * NB + b) * kBlockBytes + kk * 32;
                            const uint32_t ax2 = xp + (1 * NB + b) * kBlockBytes + kk * 32;
                            mma_f16(dS, smem_desc(ax, 16, 1024, kSwz128),
                                    smem_desc(w1 + kk * 32, 16, 1024, kSwz128), idesc_e, acc);
                            acc = 1;
                            mma_f16(dS, smem_desc(ax2, 16, 1024, kSwz128),
                                    smem_desc(w2 + kk * 32, 16, 1024, kSwz128), idesc_e, 1);
                        }
                        mma_commit(&bars->wempty[s1]);
                        mma_commit(&bars->wempty[s2]);
                    }
                    if (!ok) break;
                    mma_commit(MODE == kLse ? &bars->sfull[buf] : &bars->sfull[0]);
                }
                if (!ok) break;
                if (MODE != kLse) {
                    // M-step: D[comp, col] += R^T[comp, pt] * XX[pt, col]
                    if (!mbar_wait(&bars->rfull, it & 1, err, abort_flag)) break;
                    tc_fence_after();
                    const uint32_t rb = smem_u32(sm + S::RING);          // r_hi blocks
                    const uint32_t rl = rb + 2 * kBlockBytes;            // r_lo blocks
                    const uint32_t ones = smem_u32(sm + S::ONES);
                    const uint32_t id_full = idesc_f16(128, 2 * D, true, true);
                    const uint32_t id_half = idesc_f16(128, D, true, true);
                    const uint32_t id_s0 = idesc_f16(128, 16, true, false);
                    for (int kk = 0; kk < kTileP / 16; ++kk) {
                        const uint64_t a_hi = smem_desc(rb + kk * 2048, kBlockBytes, 1024, kSwz128);
                        const uint64_t a_lo = smem_desc(rl + kk * 2048, kBlockBytes, 1024, kSwz128);
                        const uint64_t b_hi = smem_desc(xp + kk * 2048, kBlockBytes, 1024, kSwz128);
                        const uint32_t acc = first_m ? 0u : 1u;
                        mma_f16(t_st, a_hi, b_hi, id_full, acc);
                        if (XEXACT) {
                            const uint64_t b_sq_lo =
                                smem_desc(xp + 3 * NB * kBlockBytes + kk * 2048, kBlockBytes, 1024, kSwz128);
                            mma_f16(t_st + D, a_hi, b_sq_lo, id_half, 1);
                        } else {
                            const uint64_t b_lo =
                                smem_desc(xp + 2 * NB * kBlockBytes + kk * 2048, kBlockBytes, 1024, kSwz128);
                            mma_f16(t_st, a_hi, b_lo, id_full, 1);
                        }
                        mma_f16(t_st, a_lo, b_hi, id_full, 1);
                        const uint64_t b_one = smem_desc(ones + (kk & 3) * 32 + (kk >> 2) * 2048, 16, 1024, kSwz128);
                        mma_f16(t_s0, a_hi, b_one, id_s0, acc);
                        mma_f16(t_s0, a_lo, b_one, id_s0, 1);
                        first_m = false;
                    }
                }
                mma_commit(&bars->xfree);
            }
            mma_commit(&bars->done);
            mbar_wait_drain(&bars->done, 0, err);   // no MMA in flight at teardown
        }
    } else if (warp >= 8) {
        // ===================== X tile converter (256 threads)
        const int ct = tid - 256;
        constexpr int CPR = D / 8;                   // 16-byte chunks per row
        constexpr int GROUPS = kTileP * CPR / 256;   // chunks per thread
        int it = 0;
        for (int64_t t = t_begin; t < t_end; t += t_step, ++it) {
            float v[GROUPS][8];
#pragma unroll
            for (int i = 0; i < GROUPS; ++i) {
                const int gi = ct + 256 * i;
                const int p = gi / CPR, c = gi % CPR;
                const int64_t n = t * kTileP + p;
                if (n < N) {
                    load8<XT>(X + n * D + c * 8, v[i]);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[i][e] = 0.f;
                }
            }
            if (it > 0 && !mbar_wait(&bars->xfree, (it - 1) & 1, err, abort_flag)) break;
            bool bad = false;
#pragma unroll
            for (int i = 0; i < GROUPS; ++i) {
                const int gi = ct + 256 * i;
                const int p = gi / CPR, c = gi % CPR;
                const int b = c / 8, cc = c % 8;
                uint32_t w_hi[4], w_lo[4], w_sh[4], w_sl[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    float x0 = v[i][e], x1 = v[i][e + 1];
                    bad |= !(fabsf(x0) < kRangeMax) || !(fabsf(x1) < kRangeMax);
                    __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
                    __half l0 = __float2half_rn(x0 - __half2float(h0));
                    __half l1 = __float2half_rn(x1 - __half2float(h1));
                    float s0 = x0 * x0, s1 = x1 * x1;
                    __half sh0 = __float2half_rn(s0), sh1 = __float2half_rn(s1);
                    __half sl0 = __float2half_rn(s0 - __half2float(sh0));
                    __half sl1 = __float2half_rn(s1 - __half2float(sh1));
                    w_hi[e / 2] = pack_half2(h0, h1);
                    w_lo[e / 2] = pack_half2(l0, l1);
                    w_sh[e / 2] = pack_half2(sh0, sh1);
                    w_sl[e / 2] = pack_half2(sl0, sl1);
                }
                const uint32_t off = swz128_off(p, cc);
                *reinterpret_cast<uint4 *>(sm + (0 * NB + b) * kBlockBytes + off) =
                    make_uint4(w_hi[0], w_hi[1], w_hi[2], w_hi[3]);
                *reinterpret_cast<uint4 *>(sm + (1 * NB + b) * kBlockBytes + off) =
                    make_uint4(w_sh[0], w_sh[1], w_sh[2], w_sh[3]);
                *reinterpret_cast<uint4 *>(sm + (2 * NB + b) * kBlockBytes + off) =
                    make_uint4(w_lo[0], w_lo[1], w_lo[2], w_lo[3]);
                *reinterpret_cast<uint4 *>(sm + (3 * NB + b) * kBlockBytes + off) =
                    make_uint4(w_sl[0], w_sl[1], w_sl[2], w_sl[3]);
            }
            if (__any_sync(0xffffffffu, bad) && lane == 0) set_error(err, GMM_ERR_RANGE);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->xfull);
        }
    } else if (warp >= 4) {
        // ===================== TMEM readers: scores -> responsibilities / LSE
        const int p = tid - 128;                          // TMEM lane = point row
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        uint32_t q = 0;
        int it = 0;
        for (int64_t t = t_begin; t < t_end; t += t_step, ++it) {
            const int64_t n = t * kTileP + p;
            const bool valid = n < N;
            if (MODE == kLse) {
                float m = -INFINITY, l = 0.f;             // in log2 units
                bool ok = true;
                for (int c = 0; c < nchunks; ++c, ++q) {
                    const uint32_t buf = q & 1;
                    if (!mbar_wait(&bars->sfull[buf], (q >> 1) & 1, err, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    for (int cc = 0; cc < C / 32; ++cc) {
                        uint32_t r[32];
                        tmem_ld32(tmem + lane_base + buf * C + cc * 32, r);
                        tmem_ld_wait();
                        const int kb = c * kChunk1 + cc * 32;
                        float y[32], cm = -INFINITY;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            y[i] = fmaf(__uint_as_float(r[i]), __ldg(P.ak + kb + i),
                                        __ldg(P.bk + kb + i));
                            cm = fmaxf(cm, y[i]);
                        }
                        const float nm = fmaxf(m, cm);
                        if (nm != -INFINITY) {
                            float s = 0.f;
#pragma unroll
                            for (int i = 0; i < 32; ++i) s += exp2f(y[i] - nm);
                            l = l * exp2f(m - nm) + s;
                            m = nm;
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->sfree[buf]);
                }
                if (!ok) break;
                const float lse = (m + log2f(l)) * 0.69314718055994531f;
                if (valid) {
                    if (!(m > -INFINITY)) set_error(err, GMM_ERR_NONFINITE);
                    lse_out[n] = lse;
                    if (loglik) loglik[n] = lse;
                }
                // fp64 tile sum in fixed order: lane sums, then warps 0..3
                double ds = valid ? (double)lse : 0.0;
#pragma unroll
                for (int o = 16; o; o >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, o);
                double *llw_d = reinterpret_cast<double *>(llw);
                if (lane == 0) llw_d[warp & 3] = ds;
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (p == 0) ll_part[t] = (llw_d[0] + llw_d[1]) + (llw_d[2] + llw_d[3]);
                asm volatile("bar.sync 1, 128;" ::: "memory");
            } else {
                if (!mbar_wait(&bars->sfull[0], it & 1, err, abort_flag)) break;
                tc_fence_after();
                float lse2;   // l_n in log2 units
                if (MODE == kSingle) {
                    float m = -INFINITY, l = 0.f;
                    for (int cc = 0; cc < kSlice / 32; ++cc) {
                        uint32_t r[32];
                        tmem_ld32(tmem + lane_base + cc * 32, r);
                        tmem_ld_wait();
                        float y[32], cm = -INFINITY;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            y[i] = fmaf(__uint_as_float(r[i]), cA[cc * 32 + i], cB[cc * 32 + i]);
                            cm = fmaxf(cm, y[i]);
                        }
                        const float nm = fmaxf(m, cm);
                        if (nm != -INFINITY) {
                            float s = 0.f;
#pragma unroll
                            for (int i = 0; i < 32; ++i) s += exp2f(y[i] - nm);
                            l = l * exp2f(m - nm) + s;
                            m = nm;
                        }
                    }
                    lse2 = m + log2f(l);
                    const float lse = lse2 * 0.69314718055994531f;
                    if (valid) {
                        if (!(m > -INFINITY)) set_error(err, GMM_ERR_NONFINITE);
                        if (loglik) loglik[n] = lse;
                    }
                    double ds = valid ? (double)lse : 0.0;
#pragma unroll
                    for (int o = 16; o; o >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, o);
                    double *llw_d = reinterpret_cast<double *>(llw);
                    if (lane == 0) llw_d[warp & 3] = ds;
                    asm volatile("bar.sync 1, 128;" ::: "memory");
                    if (p == 0) ll_part[t] = (llw_d[0] + llw_d[1]) + (llw_d[2] + llw_d[3]);
                    asm volatile("bar.sync 1, 128;" ::: "memory");
                } else {
                    lse2 = valid ? lse_in[n] * kLog2e : INFINITY;
                }
                if (!valid) lse2 = INFINITY;   // r = 0 for padding rows
                // Per-component dynamic scale.  r_nk spans many orders of
                // magnitude (a component far from every point of the data
                // has only tiny responsibilities), while fp16 pieces keep
                // 22 bits only near their top exponent.  So component k's
                // responsibilities enter the M-step as r' = r * 2^sig_k,
                // with sig_k chosen from the largest r of k seen so far
                // (its max r' sits in [2^14, 2^15]); when a later tile
                // lowers sig_k, the TMEM statistics row k is rescaled by the
                // same power of two (exact), as an online softmax rescales
                // its output.  The fp64 reduction divides the scale out.
                // Pass A: max over the tile's points of ceil(log2 r_nk).
                for (int cc = 0; cc < kSlice / 32; ++cc) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_base + cc * 32, r);
                    tmem_ld_wait();
                    int mine = -250;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float e = fmaf(__uint_as_float(r[i]), cA[cc * 32 + i],
                                             cB[cc * 32 + i]) - lse2;
                        const int ce = (int)ceilf(fmaxf(e, -250.f));
                        const int m = __reduce_max_sync(0xffffffffu, ce);
                        if (lane == i) mine = m;
                    }
                    tmax[(warp & 3) * kSlice + cc * 32 + lane] = mine;
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
                {
                    // thread p owns component p's scale and TMEM statistics row
                    int tm = max(max(tmax[p], tmax[kSlice + p]),
                                 max(tmax[2 * kSlice + p], tmax[3 * kSlice + p]));
                    const int s_old = (it == 0) ? kSigInit : sig[p];
                    const int s_new = min(s_old, 15 - tm);
                    sig[p] = s_new;
                    const int delta = s_new - s_old;
                    if (it > 0 && __any_sync(0xffffffffu, delta < 0)) {
                        // statistics are idle here (the previous M-step has
                        // completed before this tile's scores); rescale rows
                        const float f = exp2f((float)delta);
                        uint32_t r[32];
                        tmem_ld32(t_s0 + lane_base, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
                        tmem_st32(t_s0 + lane_base, r);
                        for (int cc = 0; cc < 2 * D / 32; ++cc) {
                            tmem_ld32(t_st + lane_base + cc * 32, r);
                            tmem_ld_wait();
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
                            tmem_st32(t_st + lane_base + cc * 32, r);
                        }
                        tmem_st_wait();
                    }
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
                // Pass B: r'_nk = 2^(y_nk - l_n + sig_k) -> r_hi / r_lo
                // (MN-major, SWIZZLE_128B)
                uint8_t *rhi = sm + S::RING;
                uint8_t *rlo = rhi + 2 * kBlockBytes;
                for (int cc = 0; cc < kSlice / 32; ++cc) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_base + cc * 32, r);
                    tmem_ld_wait();
                    uint32_t ph[16], pl[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        float y0 = fmaf(__uint_as_float(r[i]), cA[cc * 32 + i], cB[cc * 32 + i]) -
                                   lse2 + (float)sig[cc * 32 + i];
                        float y1 = fmaf(__uint_as_float(r[i + 1]), cA[cc * 32 + i + 1],
                                        cB[cc * 32 + i + 1]) - lse2 + (float)sig[cc * 32 + i + 1];
                        float r0 = exp2f(y0), r1 = exp2f(y1);
                        __half h0 = __float2half_rn(r0), h1 = __float2half_rn(r1);
                        __half l0 = __float2half_rn(r0 - __half2float(h0));
                        __half l1 = __float2half_rn(r1 - __half2float(h1));
                        ph[i / 2] = pack_half2(h0, h1);
                        pl[i / 2] = pack_half2(l0, l1);
                    }
                    const int blk = cc / 2;                 // 64-component block
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int chunk = (cc & 1) * 4 + j;   // 16-byte chunk within the 128-B row
                        const uint32_t off = blk * kBlockBytes + swz128_off(p, chunk);
                        *reinterpret_cast<uint4 *>(rhi + off) =
                            make_uint4(ph[4 * j], ph[4 * j + 1], ph[4 * j + 2], ph[4 * j + 3]);
                        *reinterpret_cast<uint4 *>(rlo + off) =
                            make_uint4(pl[4 * j], pl[4 * j + 1], pl[4 * j + 2], pl[4 * j + 3]);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->rfull);
            }
        }
        if (MODE != kLse) {
            // drain the slice's statistics: lane = component row
            if (mbar_wait(&bars->done, 0, err, abort_flag)) {
                tc_fence_after();
                const int k = comp0 + p;
                const size_t width = (size_t)K * (1 + 2 * (size_t)D);
                float *out = partial + (size_t)blockIdx.y * width;
                uint32_t r[32];
                const bool any = t_begin < t_end;   // a CTA without tiles writes zeros
                tmem_ld32(t_s0 + lane_base, r);
                tmem_ld_wait();
                if (k < K) {
                    out[k] = any ? __uint_as_float(r[0]) : 0.f;
                    partial_sig[(size_t)blockIdx.y * K + k] = any ? sig[p] : 0;
                }
                for (int cc = 0; cc < 2 * D / 32; ++cc) {
                    tmem_ld32(t_st + lane_base + cc * 32, r);
                    tmem_ld_wait();
                    if (k < K) {
                        const int col0 = cc * 32;
                        float *dst = (col0 < D) ? out + K + (size_t)k * D + col0
                                                : out + K + (size_t)K * D + (size_t)k * D + (col0 - D);
#pragma unroll
                        for (int i = 0; i < 32; ++i) dst[i] = any ? __uint_as_float(r[i]) : 0.f;
                    }
                }
            }
        }
    }

    // ---- teardown: every role has left its loop (all waits are bounded)
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- host side

namespace {

int tc_kp(int K) { return K <= kSlice ? kSlice : (K + kChunk1 - 1) / kChunk1 * kChunk1; }

bool tc_shape_ok(gmm_dtype dt, int d, int K) {
    (void)dt;
    return (d == 64 || d == 128) && K >= 1 && K <= 4096 * 4;
}

int tc_sm_count() {
    static int cached = 0;
    if (!cached) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&cached, cudaDevAttrMultiProcessorCount, dev);
        if (cached <= 0) cached = 148;
    }
    return cached;
}

constexpr int kMaxRanges = 148;

}  // namespace

bool gmm_tc_supported(gmm_dtype dt, int64_t N, int d, int K, uint32_t flags) {
    (void)N;
    (void)flags;
    return tc_shape_ok(dt, d, K);
}

int gmm_tc_regime(gmm_dtype dt, int64_t N, int d, int K, uint32_t flags) {
    (void)dt; (void)N; (void)d;
    if (K > kSlice || (flags & GMM_FLAG_FORCE_TWO_SWEEP)) return 2;
    return 1;
}

size_t gmm_tc_ws_bytes(int64_t N, int d, int K) {
    (void)N;
    if (d % 64 != 0) return 0;
    int Kp = tc_kp(K);
    if (Kp < kChunk1) Kp = kChunk1;   // the two-sweep flag pads to a 256 multiple
    return align_up(img_bytes(Kp, d / 64)) + 2 * align_up((size_t)Kp * 4);
}

int64_t gmm_tc_max_partials(int64_t N, int d, int K) {
    (void)N; (void)d; (void)K;
    return kMaxRanges;
}

int64_t gmm_tc_max_ll(int64_t N, int d, int K) {
    (void)d; (void)K;
    return (N + kTileP - 1) / kTileP;
}

template <int NB, typename XT, int MODE>
static cudaError_t launch_fused(dim3 grid, const XT *X, int64_t N, int K, const TcParams &P,
                                const GmmWs &w, float *loglik, int64_t tiles_per_range,
                                cudaStream_t s) {
    auto kern = gmm_tc_fused_kernel<NB, XT, MODE>;
    const int smem = Smem<NB, MODE>::TOTAL;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, s>>>(X, N, K, P, w.lse, w.lse, loglik, w.ll_part, w.partial,
                                      w.psig, tiles_per_range, w.err);
    return cudaGetLastError();
}

template <int NB, typename XT>
static cudaError_t launch_tc_t(const XT *X, int64_t N, int K, const TcParams &P, const GmmWs &w,
                               float *loglik, bool two_sweep, int *num_partials, int64_t *num_ll,
                               cudaStream_t s) {
    const int64_t ntiles = (N + kTileP - 1) / kTileP;
    const int slices = P.Kp / kSlice;
    int ranges = kMaxRanges / (two_sweep ? slices : 1);
    if (ranges < 1) ranges = 1;
    if (ranges > ntiles) ranges = (int)ntiles;
    const int64_t tpr = (ntiles + ranges - 1) / ranges;
    ranges = (int)((ntiles + tpr - 1) / tpr);
    *num_partials = ranges;
    *num_ll = ntiles;
    cudaError_t e;
    timer_begin(s);
    if (two_sweep) {
        int g1 = tc_sm_count();
        if (g1 > ntiles) g1 = (int)ntiles;
        e = launch_fused<NB, XT, kLse>(dim3(g1), X, N, K, P, w, loglik, 0, s);
        if (e != cudaSuccess) return e;
        e = launch_fused<NB, XT, kStats>(dim3(slices, ranges), X, N, K, P, w, nullptr, tpr, s);
        note_launches(2);
    } else {
        e = launch_fused<NB, XT, kSingle>(dim3(1, ranges), X, N, K, P, w, loglik, tpr, s);
        note_launches(1);
    }
    timer_end(s);
    return e;
}

cudaError_t launch_gmm_tc(const void *X, gmm_dtype dt, int64_t N, int d, int K,
                          const float *means, const float *vars, const float *logw,
                          const GmmWs &w, float *loglik, uint32_t flags, int *num_partials,
                          int64_t *num_ll, cudaStream_t s) {
    if (!tc_shape_ok(dt, d, K)) return cudaErrorNotSupported;
    const bool two = gmm_tc_regime(dt, N, d, K, flags) == 2;
    int Kp = tc_kp(K);
    if (two && Kp < kChunk1) Kp = kChunk1;
    const int NB = d / 64;
    uint8_t *img = (uint8_t *)w.tc;
    float *ak = (float *)((char *)w.tc + align_up(img_bytes(Kp, NB)));
    float *bk = (float *)((char *)ak + align_up((size_t)Kp * 4));
    gmm_tc_params_kernel<<<(Kp * 32 + 255) / 256, 256, 0, s>>>(means, vars, logw, K, d, Kp, img,
                                                               ak, bk, w.err);
    note_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    TcParams P{img, ak, bk, Kp};
#define GMM_TC_CASE(NBV, T)                                                                    \
    return launch_tc_t<NBV, T>((const T *)X, N, K, P, w, loglik, two, num_partials, num_ll, s)
    if (NB == 2) {
        if (dt == GMM_F32) GMM_TC_CASE(2, float);
        if (dt == GMM_BF16) GMM_TC_CASE(2, __nv_bfloat16);
        GMM_TC_CASE(2, __half);
    } else {
        if (dt == GMM_F32) GMM_TC_CASE(1, float);
        if (dt == GMM_BF16) GMM_TC_CASE(1, __nv_bfloat16);
        GMM_TC_CASE(1, __half);
    }
#undef GMM_TC_CASE
}

}  // namespace gmmb
