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
// Warp roles (320 threads): warp 0 streams the parameter pieces (1-D bulk
// copies into a ring), warp 1 issues tcgen05.mma, warps 2-9 convert X tiles
// into the fp16 pieces and read TMEM (scores, then the statistics).  All
// waits are bounded (tc::mbar_wait).
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
constexpr int kThreads = 320;  // 10 warps (see the role list at the kernel)
constexpr int kBlockBytes = kTileP * 128;  // one 64-feature block of a 128-row tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRangeMax = 181.0f;        // 181^2 < 65504 (fp16 max)
// Initial responsibility scale exponent: r < 2^-100 never matters (such a
// component has N_k < 1e-12 N for any N below 2^60 and is kept as it was).
constexpr int kSigInit = 115;

enum Mode { kLse = 0, kStats = 1, kSingle = 2, kAssign = 3 };
// Sweep 1 (the per-point log-sum-exp over 256-component chunks) and the soft
// assignment, which is sweep 1 plus a per-point top-r selection, share every
// structural choice.
__host__ __device__ constexpr bool sweep1(int mode) { return mode == kLse || mode == kAssign; }

// Outputs of the soft assignment (kAssign): per point the kTopMax best
// components kept on chip; the first R (R <= kTopMax) with r_nk >= tau are
// written as ids [N x R] / resp [N x R] (id -1, resp 0 past the cut).
struct AssignOut {
    int R;
    float tau;
    int32_t *ids;
    float *resp;
    const int *dlist;     // direct-form components and their [slot x N] scores
    const float *dscore;  // (log2 units)
};

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
    // Components scored in the direct form (gmm_tc_direct_scores_kernel) are
    // left out here (a_k = 0, b_k = -inf); when *dcount > 0, dmf[n] holds
    // (max, sum) of their 2^(score) terms for point n, merged into l_n.
    const float2 *dmf;
    const int *dcount;
    // X enters the tensor core as x * 2^-s (an exact power of two chosen by
    // the max|x| scan and gmm_tc_params_kernel so that |x| 2^-s < 181 and
    // x^2 stays inside the fp16 range); the W pieces carry 2^s and 2^2s, and
    // the statistics leave TMEM multiplied back by 2^s (S1) and 2^2s (S2).
    const int *xs_exp;
    // Testing only (GMM_FLAG_TEST_STALL): the parameter producer of CTA
    // (0, 0) withholds its pipeline stage number `stall` (never issues it), so
    // the MMA issuer's bounded wait for it runs out; -1 = off.
    int stall;
};

// Ill-conditioning of the expanded score form.  For a point near component
// k the terms x W1, x^2 W2 and c_k are each of size about
// Q_k = sum_j mu_kj^2 / var_kj while their sum is O(d), and the tensor
// core's fp32 accumulation truncates at that magnitude: the absolute score
// error grows like 2^-21 Q_k.  Components above kCondHard (a component that
// collapsed onto a point: var at the floor, Q ~ 1e8) must be scored in the
// direct form s = c_k + sum_j nhl_kj (x_j - mu_kj)^2 on CUDA cores; those
// above kCondSoft take the direct form while slots remain (direct_slots(K)
// per call, hard ones first).  More hard components than slots:
// GMM_ERR_RANGE.
constexpr double kCondSoft = 4096.0;
constexpr double kCondHard = 16384.0;
constexpr int kDirectMax = 512;   // the most slots any K gets

// Direct-form slots for K components: 64, K/16 for 1024 < K <= 2048, and K/8
// above, at most kDirectMax.  At K = 4096 on data drawn from a 4096-component
// mixture, EM makes ~230 components hard and ~200 more soft by its third
// iteration (counted with the oracle on a 200,000-point prefix); a soft
// component left in the expanded form carries score errors up to ~2^-7,
// which a point with |l_n| near 1 turns into a 1e-3 relative log-likelihood
// error.  The workspace holds [slots x C] fp32 scores for a chunk of C
// points (gmm_tc_chunk_points).
__host__ __device__ inline int direct_slots(int K) {
    const int want = K > 2048 ? K / 8 : (K / 16 > 64 ? K / 16 : 64);
    const int cap = want < kDirectMax ? want : kDirectMax;
    return K < cap ? K : cap;
}

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
// The exponent s of the X scale 2^-s: the one power of two with
// max|x| 2^-s in [90.5, 181), so x^2 stays inside the fp16 range and the
// data's small values keep as many fp16 bits as the range allows (the fp16
// pieces of x^2 have an absolute floor of 2^-25, which data held near
// |x| ~ 1 would otherwise waste: x = 1e-3 has x^2 below the normal range).
// s may be negative.  0 when max|x| is 0 or not finite (the converters then
// report the non-finite values); s >= -100.
__device__ __forceinline__ int x_scale_exp(uint32_t max_bits) {
    const float mx = __uint_as_float(max_bits);
    if (!(mx < INFINITY) || !(mx > 0.f)) return 0;
    int e = 0;
    frexp((double)mx / (double)kRangeMax, &e);   // mx / 181 < 2^e
    while ((double)mx * ldexp(1.0, -e) >= (double)kRangeMax) ++e;
    while (e > -100 && (double)mx * ldexp(1.0, -(e - 1)) < (double)kRangeMax) --e;
    return e < -100 ? -100 : e;
}

// max |x| as the bits of a non-negative float: an integer max, so the result
// does not depend on the order of the atomics (NaN sorts above +inf).  The
// scan is folded into the direct-form scores kernel's pass over X.
__device__ __forceinline__ uint32_t abs_bits(float v) { return __float_as_uint(v) & 0x7fffffffu; }

// Grid-stride scan of X for max |x| (thread `t` of `nt`).
template <typename XT>
__device__ uint32_t xmax_scan(const XT *__restrict__ X, int64_t n_elems, int64_t t, int64_t nt) {
    constexpr int V = 16 / sizeof(XT);
    const int64_t nvec = n_elems / V;
    uint32_t m = 0;
    for (int64_t i = t; i < nvec; i += nt) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(X) + i);
        const XT *e8 = reinterpret_cast<const XT *>(&u);
#pragma unroll
        for (int e = 0; e < V; ++e) m = max(m, abs_bits(to_float(e8[e])));
    }
    for (int64_t i = nvec * V + t; i < n_elems; i += nt) m = max(m, abs_bits(to_float(X[i])));
    return m;
}

// The block's max into *max_bits (which is 0 before the first block adds to
// it).  Every thread of the block calls it; blockDim.x <= 1024.
__device__ void block_max_to(uint32_t m, uint32_t *max_bits) {
    __shared__ uint32_t wm[32];
    m = __reduce_max_sync(0xffffffffu, m);
    __syncthreads();   // (wm may still be read by a previous call's thread 0)
    if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) b = max(b, wm[w]);
        if (b) atomicMax(max_bits, b);
    }
}

// a1, first part (nothing here depends on the data): per component the
// expanded form's constant b_k = c_k log2(e), c_k = log w_k -
// 1/2 sum_j (mu^2/var + log(2 pi var)), the conditioning Q_k -> dflag (2 hard,
// 1 soft, 0 fine; a dead component is never listed), and the parameter
// checks: a parameter that is not finite, a variance <= 0 or a log weight
// that is NaN or +inf records GMM_ERR_NONFINITE.  One warp per component,
// sums in fp64 in a fixed butterfly order.
__global__ void gmm_tc_cond_kernel(const float *__restrict__ means, const float *__restrict__ vars,
                                   const float *__restrict__ logw, int K, int d, int Kp,
                                   float *__restrict__ bk, int *__restrict__ dflag, int *err) {
    const int k = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    if (k >= Kp) return;
    if (k >= K) {
        if (lane == 0) { bk[k] = -INFINITY; dflag[k] = 0; }
        return;
    }
    double cacc = 0.0, qk = 0.0;
    bool bad = lane == 0 && (isnan(logw[k]) || logw[k] == INFINITY);
    for (int j = lane; j < d; j += 32) {
        double mu = means[(size_t)k * d + j], v = vars[(size_t)k * d + j];
        bad |= !isfinite(mu) || !isfinite(v) || !(v > 0.0);
        cacc += mu * mu / v + log(2.0 * M_PI * v);
        qk += mu * mu / v;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        cacc += __shfl_xor_sync(0xffffffffu, cacc, o);
        qk += __shfl_xor_sync(0xffffffffu, qk, o);
    }
    if (bad) set_error(err, GMM_ERR_NONFINITE);
    if (lane == 0) {
        const double c = (double)logw[k] - 0.5 * cacc;
        bk[k] = (float)(c * (double)kLog2e);
        dflag[k] = (logw[k] == -INFINITY) ? 0 : (qk > kCondHard ? 2 : (qk > kCondSoft ? 1 : 0));
    }
}

// a1, second part (after max|x|): the X scale, and per component the W
// pieces of the parameter image with their power-of-two scale 2^-e_k and
// a_k = 2^e_k log2(e); a component listed for the direct form (dflag 3)
// gets a_k = 0 (its b_k is already -inf).
__global__ void gmm_tc_params_kernel(const float *__restrict__ means,
                                     const float *__restrict__ vars, int K, int d, int Kp,
                                     const uint32_t *__restrict__ xmax, int *__restrict__ xs_exp,
                                     uint8_t *__restrict__ img, float *__restrict__ ak,
                                     const int *__restrict__ dflag, int *err) {
    const int warp = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    if (warp >= Kp) return;
    // X scale: W1 multiplies x 2^-s and W2 multiplies x^2 2^-2s.  The scan's
    // max also decides the data's range for every converter: with the scale,
    // no value can leave the fp16 range, and NaN / Inf in X is reported here.
    const uint32_t xmb = *xmax;
    const int xs = x_scale_exp(xmb);
    if (warp == 0 && lane == 0) {
        *xs_exp = xs;
        if (xmb >= 0x7f800000u) set_error(err, GMM_ERR_NONFINITE);
    }
    const double ws1 = ldexp(1.0, xs), ws2 = ldexp(1.0, 2 * xs);
    const int k = warp;
    const int NB = (d + 63) / 64;   // d < 64 is padded to one 64-feature block
    if (k >= K) {
        for (int j = lane; j < NB * 64; j += 32)
            for (int pc = 0; pc < 4; ++pc)
                *reinterpret_cast<__half *>(img + img_elem(pc, j / 64, k, j % 64, NB, Kp)) =
                    __float2half_rn(0.f);
        if (lane == 0) ak[k] = 0.f;
        return;
    }
    // max |W| for the scale (the parameters were checked by gmm_tc_cond_kernel)
    double mx = 0.0;
    for (int j = lane; j < d; j += 32) {
        double mu = means[(size_t)k * d + j], v = vars[(size_t)k * d + j];
        double w1 = mu / v * ws1, w2 = -0.5 / v * ws2;
        mx = fmax(mx, fmax(fabs(w1), fabs(w2)));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    int ex = 0;
    frexp(mx, &ex);          // mx < 2^ex
    const int e = ex - 8;    // |W| * 2^-e < 2^8
    const double inv = ldexp(1.0, -e);
    if (!(mx > 0.0) || !isfinite(mx)) set_error(err, GMM_ERR_RANGE);
    for (int j = lane; j < NB * 64; j += 32) {
        const bool real = j < d;   // padded features have zero pieces
        double mu = real ? means[(size_t)k * d + j] : 0.0, v = real ? vars[(size_t)k * d + j] : 1.0;
        double w[2] = {real ? mu / v * ws1 * inv : 0.0, real ? -0.5 / v * ws2 * inv : 0.0};
        for (int t = 0; t < 2; ++t) {
            __half hi = __float2half_rn((float)w[t]);
            __half lo = __float2half_rn((float)(w[t] - (double)__half2float(hi)));
            *reinterpret_cast<__half *>(img + img_elem(2 * t, j / 64, k, j % 64, NB, Kp)) = hi;
            *reinterpret_cast<__half *>(img + img_elem(2 * t + 1, j / 64, k, j % 64, NB, Kp)) = lo;
        }
    }
    if (lane == 0) ak[k] = dflag[k] == 3 ? 0.f : (float)(ldexp(1.0, e) * (double)kLog2e);
}

// a1': the list of direct-form components: every hard one (flag 2) and the
// soft ones (flag 1) in increasing k while slots remain; slots are assigned
// in increasing k, so nothing depends on scheduling.  A listed component
// gets a_k = 0, b_k = -inf, which removes it from the tensor-core sums.
// One block of 1024 threads.
__global__ void __launch_bounds__(1024)
gmm_tc_direct_list_kernel(int *__restrict__ dflag, int Kp, int cap, float *__restrict__ bk,
                          int *__restrict__ dlist, int *__restrict__ dcount, int *err) {
    __shared__ int part[2][1024];
    const int t = threadIdx.x;
    const int per = (Kp + 1023) / 1024;
    const int b = min(Kp, t * per), e = min(Kp, b + per);
    // pass 1: hard and soft counts -> which soft components get a slot
    int ch = 0, cs = 0;
    for (int k = b; k < e; ++k) { ch += dflag[k] == 2; cs += dflag[k] == 1; }
    part[0][t] = ch;
    part[1][t] = cs;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {   // inclusive scans
        const int vh = t >= o ? part[0][t - o] : 0, vs = t >= o ? part[1][t - o] : 0;
        __syncthreads();
        part[0][t] += vh;
        part[1][t] += vs;
        __syncthreads();
    }
    const int hard = part[0][1023];
    const int soft_room = cap > hard ? cap - hard : 0;
    int rs = part[1][t] - cs;   // soft rank of this thread's first soft component
    int cl = 0;
    for (int k = b; k < e; ++k) {
        const int f = dflag[k];
        cl += (f == 2) || (f == 1 && rs < soft_room);
        rs += f == 1;
    }
    __syncthreads();
    part[0][t] = cl;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
        const int v = t >= o ? part[0][t - o] : 0;
        __syncthreads();
        part[0][t] += v;
        __syncthreads();
    }
    // pass 2: slots in increasing k
    int sl = part[0][t] - cl;
    rs = part[1][t] - cs;
    for (int k = b; k < e; ++k) {
        const int f = dflag[k];
        const bool listed = (f == 2) || (f == 1 && rs < soft_room);
        rs += f == 1;
        if (listed) {
            if (sl < cap) dlist[sl] = k;
            ++sl;
            dflag[k] = 3;   // (gmm_tc_params_kernel then writes a_k = 0)
            bk[k] = -INFINITY;
        }
    }
    if (t == 1023) {
        *dcount = min(part[0][1023], cap);
        if (hard > cap) set_error(err, GMM_ERR_RANGE);
    }
}

namespace {

// Shared-memory plan of the fused kernel (bytes, offsets from a 1024-aligned base).
template <int NB, int MODE>
struct Smem {
    static constexpr int C = sweep1(MODE) ? kChunk1 : kSlice;     // components per chunk
    static constexpr int XP = 4 * NB * kBlockBytes;               // X pieces
    static constexpr int STAGE = C * 128;                         // one parameter stage
    static constexpr int NSTAGE = sweep1(MODE) ? 3 : 5;
    static constexpr int RING = XP;                               // ring offset
    static constexpr int RBYTES = 2 * 2 * kBlockBytes;            // r_hi, r_lo (2 comp blocks)
    static constexpr int ONES = RING + NSTAGE * STAGE;            // 16 x 128 fp16 ones
    static constexpr int ONES_BYTES = sweep1(MODE) ? 0 : 4096;
    // constants: sweep 1: (m, l) of the second column half [128 x 2];
    // otherwise a_k, b_k [2 x 128], per-quadrant tile maxima [4 x 128],
    // scales [128], (m, l) of both halves [2 x 128 x 2]
    static constexpr int CONSTS = ONES + ONES_BYTES;
    static constexpr int CONSTS_BYTES = sweep1(MODE) ? 1024 : 11 * kSlice * 4;
    static constexpr int BARS = CONSTS + CONSTS_BYTES;
    static constexpr int BARS_BYTES = 256;
    static constexpr int MISC = BARS + BARS_BYTES;                // tmem addr, abort, ll scratch
    static constexpr int TOTAL = MISC + 256 + 1024;               // + alignment slack
    static_assert(sweep1(MODE) || RBYTES <= NSTAGE * STAGE, "R must fit in the ring");
    static_assert(TOTAL <= 232448, "shared memory budget");
};

// Order in which the parameter stages (one piece of one 64-feature block, for
// the chunk's components) are streamed and consumed by the E-step:
//   phase 1a, per block: [W1_hi x x_lo, fp32 inputs only], W2_hi x x2_lo
//   phase 1b, per block: W1_lo x x_hi, W2_lo x x2_hi
//   phase 2,  per block: W1_hi with x_hi and W2_hi with x2_hi together,
//             interleaved per 16-feature step.
// Phases 1a/1b add the small correction products while the accumulator is
// still small; phase 2 adds the large ones, so few additions happen at large
// magnitude (the tensor core's fp32 accumulation truncates).  Phase 1a only
// reads the lo X pieces, so it can start before the hi pieces are written.
template <int NB, bool XEXACT>
struct EProg {
    static constexpr int kP1a = XEXACT ? 1 : 2;
    static constexpr int kStages1a = NB * kP1a;
    static constexpr int kStages1 = kStages1a + 2 * NB;
    static constexpr int kStages = kStages1 + 2 * NB;
    // piece (0 W1_hi, 1 W1_lo, 2 W2_hi, 3 W2_lo), block, and the X piece it
    // multiplies in phase 1 (0 x_hi, 1 x2_hi, 2 x_lo, 3 x2_lo)
    __device__ static void stage(int i, int &pc, int &b, int &pa) {
        if (i < kStages1a) {
            b = i / kP1a;
            const bool w2 = XEXACT || (i % kP1a == 1);
            pc = w2 ? 2 : 0;
            pa = w2 ? 3 : 2;
        } else if (i < kStages1) {
            const int t = i - kStages1a;
            b = t / 2;
            pc = (t % 2 == 0) ? 1 : 3;
            pa = (t % 2 == 0) ? 0 : 1;
        } else {
            const int t = i - kStages1;
            b = t / 2;
            pc = (t % 2 == 0) ? 0 : 2;
            pa = (t % 2 == 0) ? 0 : 1;
        }
    }
};

struct Bars {
    uint64_t wfull[6], wempty[6];
    uint64_t xlo_full, xhi_full, xlo_free, xhi_free;
    uint64_t sfull[2], sfree[2];
    uint64_t rq[4];
    uint64_t rsync;   // rendezvous of the 8 reader warps
    uint64_t done;
};

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

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }

// hi = fp16(a), lo = fp16(a - hi), for a pair of values
__device__ __forceinline__ void split2(float a0, float a1, uint32_t &hi, uint32_t &lo) {
    const __half2 h = __floats2half2_rn(a0, a1);
    const float2 hf = __half22float2(h);
    hi = h2u(h);
    lo = h2u(__floats2half2_rn(a0 - hf.x, a1 - hf.y));
}

// Fold the direct-form components' (max, sum) into a point's (m, l) (log2 units).
__device__ __forceinline__ void merge_direct(float &m, float &l, float2 f) {
    const float mm = fmaxf(m, f.x);
    if (mm == -INFINITY) return;
    l = (m == -INFINITY ? 0.f : l * exp2f(m - mm)) + (f.x == -INFINITY ? 0.f : f.y * exp2f(f.x - mm));
    m = mm;
}

}  // namespace

#include "gmm_tc_direct.cuh"

namespace {
// The statistics a CTA accumulates in TMEM (fp32) are moved into its fp64
// partial row every kFlushTiles tiles and at the end.  The tensor core's fp32
// accumulation truncates, so a long accumulation chain drifts low (about
// 6e-9 relative per accumulating MMA, measured); bounding the chain at
// kFlushTiles tiles bounds that drift at about 3e-6.  The rows are scaled
// back by 2^-sig here, so the fp64 partials need no scale.
constexpr int kFlushTiles = 32;

// 2^n as a double, exactly, for |n| <= 1022.
__device__ __forceinline__ double exp2i_d(int n) {
    return __longlong_as_double((long long)(1023 + n) << 52);
}

// Move one 16-column chunk of component k's TMEM statistics into its fp64
// partial row (times `scale`), adding to what the row holds when `add`, and
// clear the chunk when `clear`.  scale == 0 writes zeros (a CTA that ran no
// M-step: its TMEM was never written).  cc < 0 is the S0 chunk (column 0 is S0);
// otherwise columns [16cc, 16cc + 16) of [S1 (D) | S2 (D)], of which the first
// DX of each half are real features.  Partial row layout, feature-major so
// that a warp's 32 components are 32 consecutive doubles:
//   S0[K] | S1[DX][K] | S2[DX][K].
// The first write of a row is a plain store, later ones are fire-and-forget
// reductions (the warp does not wait for a read); every element of a row has
// one writer thread, whose operations on it stay in program order, so the
// sums are reproducible.  Warp-collective (every lane a row).
template <int D, int DX>
__device__ __forceinline__ void flush_stats_chunk(uint32_t t_s0_row, uint32_t t_st_row, int cc,
                                                  double *out, int K, int k, double scale,
                                                  bool add, bool clear, int xs = 0) {
    const uint32_t ta = cc < 0 ? t_s0_row : t_st_row + cc * 16;
    uint32_t r[16];
    tmem_ld16(ta, r);
    tmem_ld_wait();
    // undo the X scale: S1 carries 2^-s, S2 2^-2s (exact powers of two)
    const double f = cc < 0 ? scale : scale * exp2i_d(cc * 16 < D ? xs : 2 * xs);
    auto put = [&](double *dst, uint32_t bits) {
        const double v = scale == 0.0 ? 0.0 : (double)__uint_as_float(bits) * f;
        if (add) atomicAdd(dst, v);
        else *dst = v;
    };
    if (k < K) {
        if (cc < 0) {
            put(out + k, r[0]);
        } else {
            const int col0 = cc * 16;
            const int f0 = col0 < D ? col0 : col0 - D;
            if (f0 < DX) {
                double *dst = out + K + (col0 < D ? 0 : (size_t)K * DX) + (size_t)f0 * K + k;
#pragma unroll
                for (int i = 0; i < 16; ++i) put(dst + (size_t)i * K, r[i]);
            }
        }
    }
    if (clear) {
#pragma unroll
        for (int i = 0; i < 16; ++i) r[i] = 0u;
        tmem_st16(ta, r);
    }
}
}  // namespace

#include "gmm_tc_stats.cuh"
#include "gmm_tc_cluster.cuh"
#include "gmm_tc_smallk.cuh"

// The fused kernel.  MODE kLse: grid = persistent CTAs over point tiles.
// MODE kStats / kSingle: grid = (component slices, point ranges).
//
// Roles (10 warps): warp 0 parameter producer, warp 1 MMA issuer (and TMEM
// owner), warps 2-9 workers: they convert X tiles into fp16 pieces and read
// TMEM (warp w reads lanes 32*(w%4)..+31; warps 2-5 take the first half of
// the components, 6-9 the second).
template <int NB, typename XT, int MODE, int DX>
__global__ void __launch_bounds__(kThreads, 1)
gmm_tc_fused_kernel(const XT *__restrict__ X, int64_t N, int K, TcParams P,
                    const float *__restrict__ lse_in, float *__restrict__ lse_out,
                    float *__restrict__ loglik, double *__restrict__ ll_part,
                    double *__restrict__ partial, int64_t tiles_per_range, int *err,
                    AssignOut A) {
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
    double *llw = reinterpret_cast<double *>(sm + S::MISC + 16);   // 4 per-quadrant tile sums
    float *cA = reinterpret_cast<float *>(sm + S::CONSTS);         // sweep 2 / single only
    float *cB = cA + kSlice;
    int *tmax = reinterpret_cast<int *>(cB + kSlice);               // [4][128]
    int *sig = tmax + 4 * kSlice;                                   // [128]
    float *mlx = sweep1(MODE) ? reinterpret_cast<float *>(sm + S::CONSTS)
                                : reinterpret_cast<float *>(sig + kSlice);   // (m, l) exchange

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t ntiles = (N + kTileP - 1) / kTileP;
    int64_t t_begin, t_end, t_step;
    int comp0 = 0;
    if (sweep1(MODE)) {
        t_begin = blockIdx.x; t_end = ntiles; t_step = gridDim.x;
    } else {
        comp0 = blockIdx.x * kSlice;
        t_begin = (int64_t)blockIdx.y * tiles_per_range;
        t_end = min(ntiles, t_begin + tiles_per_range);
        t_step = 1;
    }
    const int nchunks = sweep1(MODE) ? P.Kp / kChunk1 : 1;

    // ---- setup
    if (tid == 0) {
        for (int s = 0; s < S::NSTAGE; ++s) { mbar_init(&bars->wfull[s], 1); mbar_init(&bars->wempty[s], 1); }
        mbar_init(&bars->xlo_full, 8);
        mbar_init(&bars->xhi_full, 8);
        mbar_init(&bars->xlo_free, 1);
        mbar_init(&bars->xhi_free, 1);
        for (int b = 0; b < 2; ++b) { mbar_init(&bars->sfull[b], 1); mbar_init(&bars->sfree[b], 8); }
        for (int q = 0; q < 4; ++q) mbar_init(&bars->rq[q], 2);
        mbar_init(&bars->rsync, 8);
        mbar_init(&bars->done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (!sweep1(MODE)) {
        uint32_t *ones = reinterpret_cast<uint32_t *>(sm + S::ONES);   // all fp16 ones
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
    // TMEM columns: scores at 0 (two buffers of 256 in sweep 1; 128 in
    // sweep 2 / single), S0 at 128, statistics at 256 (2D columns).
    const uint32_t t_s0 = tmem + 128, t_st = tmem + 256;

    if (warp == 0) {
        // ===================== parameter-piece producer
        if (lane == 0) {
            uint32_t g = 0;
            int it = 0;
            for (int64_t t = t_begin; t < t_end && !*abort_flag; t += t_step, ++it) {
                bool r_free = sweep1(MODE) || it == 0;
                for (int c = 0; c < nchunks && !*abort_flag; ++c) {
                    const int k0 = sweep1(MODE) ? c * kChunk1 : comp0;
                    for (int i = 0; i < Prog::kStages; ++i, ++g) {
                        int pc, b, pa;
                        Prog::stage(i, pc, b, pa);
                        const int slot = g % S::NSTAGE;
                        if (g == (uint32_t)P.stall && blockIdx.x == 0 && blockIdx.y == 0)
                            continue;   // testing: this stage is withheld
                        if (!r_free && slot * S::STAGE < S::RBYTES) {
                            // this slot aliases R: the previous tile's M-step must be done
                            if (!mbar_wait(&bars->xhi_free, (it - 1) & 1, err, abort_flag))
                                goto producer_done;
                            r_free = true;
                        }
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
                if (gg == (uint32_t)P.stall && blockIdx.x == 0 && blockIdx.y == 0)
                    continue;   // never issued
                mbar_wait_drain(&bars->wfull[gg % S::NSTAGE], (gg / S::NSTAGE) & 1, err);
            }
        }
    } else if (warp == 1) {
        // ===================== MMA issuer.  One thread issues every MMA, so the
        // per-MMA work is kept to two descriptor adds: base descriptors are
        // built once, the stage program is unrolled at compile time, and the
        // ring slot advances incrementally (its issue rate bounds the tensor
        // core otherwise).
        if (lane == 0) {
            const uint32_t idesc_e = idesc_f16(128, C, false, false);
            const uint64_t dX = smem_desc(smem_u32(sm), 16, 1024, kSwz128);            // E: X pieces
            const uint64_t dR = smem_desc(smem_u32(sm + S::RING), 16, 1024, kSwz128);  // E: ring
            uint32_t slot = 0, sph = 0, q = 0;
            int it = 0;
            bool first_m = true;
            for (int64_t t = t_begin; t < t_end; t += t_step, ++it) {
                bool ok = true, have_lo = false, have_hi = false;
                for (int c = 0; c < nchunks && ok; ++c, ++q) {
                    const uint32_t buf = sweep1(MODE) ? (q & 1) : 0;
                    if (sweep1(MODE) &&
                        !mbar_wait(&bars->sfree[buf], ((q >> 1) & 1) ^ 1, err, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t dS = tmem + buf * C;
                    // phases 1a and 1b: small products
#pragma unroll
                    for (int i = 0; i < Prog::kStages1; ++i) {
                        int pc, b, pa;
                        Prog::stage(i, pc, b, pa);
                        if (!have_lo) {
                            if (!mbar_wait(&bars->xlo_full, it & 1, err, abort_flag)) { ok = false; break; }
                            have_lo = true;
                        }
                        if (pa < 2 && !have_hi) {
                            if (!mbar_wait(&bars->xhi_full, it & 1, err, abort_flag)) { ok = false; break; }
                            have_hi = true;
                        }
                        if (!mbar_wait(&bars->wfull[slot], sph, err, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        const uint64_t da = dX + (uint32_t)(((pa * NB + b) * kBlockBytes) >> 4);
                        const uint64_t db = dR + slot * (uint32_t)(S::STAGE >> 4);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_f16(dS, da + 2 * kk, db + 2 * kk, idesc_e, (i | kk) ? 1u : 0u);
                        mma_commit(&bars->wempty[slot]);
                        if (++slot == S::NSTAGE) { slot = 0; sph ^= 1; }
                    }
                    if (!ok) break;
                    if (sweep1(MODE) && c == nchunks - 1) mma_commit(&bars->xlo_free);
                    // phase 2: large products, x and x^2 terms interleaved per 16 features
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        const uint32_t s1 = slot, p1 = sph;
                        if (++slot == S::NSTAGE) { slot = 0; sph ^= 1; }
                        const uint32_t s2 = slot, p2 = sph;
                        if (++slot == S::NSTAGE) { slot = 0; sph ^= 1; }
                        if (!mbar_wait(&bars->wfull[s1], p1, err, abort_flag) ||
                            !mbar_wait(&bars->wfull[s2], p2, err, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t dax = dX + (uint32_t)(((0 * NB + b) * kBlockBytes) >> 4);
                        const uint64_t dax2 = dX + (uint32_t)(((1 * NB + b) * kBlockBytes) >> 4);
                        const uint64_t dw1 = dR + s1 * (uint32_t)(S::STAGE >> 4);
                        const uint64_t dw2 = dR + s2 * (uint32_t)(S::STAGE >> 4);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            mma_f16(dS, dax + 2 * kk, dw1 + 2 * kk, idesc_e, 1u);
                            mma_f16(dS, dax2 + 2 * kk, dw2 + 2 * kk, idesc_e, 1u);
                        }
                        mma_commit(&bars->wempty[s1]);
                        mma_commit(&bars->wempty[s2]);
                    }
                    if (!ok) break;
                    mma_commit(&bars->sfull[buf]);
                    if (sweep1(MODE) && c == nchunks - 1) mma_commit(&bars->xhi_free);
                }
                if (!ok) break;
                if (!sweep1(MODE)) {
                    // M-step: D[comp, col] += R^T[comp, pt] * XX[pt, col], one
                    // 32-point quarter at a time as the readers release it
                    const uint32_t id_full = idesc_f16(128, 2 * D, true, true);
                    const uint32_t id_half = idesc_f16(128, D, true, true);
                    const uint32_t id_s0 = idesc_f16(128, 16, true, false);
                    const uint64_t dRh = smem_desc(smem_u32(sm + S::RING), kBlockBytes, 1024, kSwz128);
                    const uint64_t dRl = dRh + (uint32_t)((2 * kBlockBytes) >> 4);
                    const uint64_t dXm = smem_desc(smem_u32(sm), kBlockBytes, 1024, kSwz128);
                    const uint64_t dOn = smem_desc(smem_u32(sm + S::ONES), 16, 1024, kSwz128);
                    const uint32_t acc_first = first_m ? 0u : 1u;
                    first_m = false;
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq) {
                        if (!mbar_wait(&bars->rq[qq], it & 1, err, abort_flag)) { ok = false; break; }
                        tc_fence_after();
#pragma unroll
                        for (int kk = 2 * qq; kk < 2 * qq + 2; ++kk) {
                            const uint64_t a_hi = dRh + (uint32_t)((kk * 2048) >> 4);
                            const uint64_t a_lo = dRl + (uint32_t)((kk * 2048) >> 4);
                            const uint64_t b_hi = dXm + (uint32_t)((kk * 2048) >> 4);
                            const uint32_t acc = (kk == 0) ? acc_first : 1u;
                            mma_f16(t_st, a_hi, b_hi, id_full, acc);
                            if (XEXACT) {
                                mma_f16(t_st + D, a_hi,
                                        dXm + (uint32_t)((3 * NB * kBlockBytes + kk * 2048) >> 4),
                                        id_half, 1u);
                            } else {
                                mma_f16(t_st, a_hi,
                                        dXm + (uint32_t)((2 * NB * kBlockBytes + kk * 2048) >> 4),
                                        id_full, 1u);
                            }
                            mma_f16(t_st, a_lo, b_hi, id_full, 1u);
                            const uint64_t b_one = dOn + (uint32_t)(((kk & 3) * 32 + (kk >> 2) * 2048) >> 4);
                            mma_f16(t_s0, a_hi, b_one, id_s0, acc);
                            mma_f16(t_s0, a_lo, b_one, id_s0, 1u);
                        }
                    }
                    if (!ok) break;
                    mma_commit(&bars->xlo_free);
                    mma_commit(&bars->xhi_free);
                }
            }
            mma_commit(&bars->done);
            mbar_wait_drain(&bars->done, 0, err);   // no MMA in flight at teardown
        }
    } else if (warp >= 2) {
        // ===================== workers (warps 2-9): X conversion and TMEM
        // reads, in an order that never waits on work that waits on them
        const int qd = warp & 3;                          // TMEM lane quadrant
        const int h = (warp - 2) >> 2;                    // component half
        const int p = qd * 32 + lane;                     // TMEM lane = point row
        const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
        uint32_t q = 0, rs = 0;
        int nflush = 0;   // times this CTA's rows went into its fp64 partial
        // bounded rendezvous of the 8 reader warps (a bar.sync could not
        // time out if another reader had left on an aborted wait)
        auto reader_sync = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->rsync);
            const bool r = mbar_wait(&bars->rsync, rs & 1, err, abort_flag);
            ++rs;
            return r;
        };
        // ---- X tile converter (all 256 worker threads): lo pieces first
        // (x_lo for fp32 inputs, x2_lo), then hi pieces
        const int ct = tid - 64;
        constexpr int CPR = DX / 8;                  // 16-byte chunks per row of X
        constexpr int GROUPS = kTileP * CPR / 256;   // chunks per thread
        static_assert(DX <= D && kTileP * CPR % 256 == 0, "feature padding");
        // features DX..D-1 of the block (d < 64) stay zero in every piece
        if constexpr (DX < D) {
            constexpr int PAD = 8 - CPR;   // zero 16-byte chunks per row
            for (int i = ct; i < kTileP * PAD * 4; i += 256) {
                const int pc = i / (kTileP * PAD), r = i % (kTileP * PAD);
                *reinterpret_cast<uint4 *>(sm + pc * NB * kBlockBytes +
                                           swz128_off(r / PAD, CPR + r % PAD)) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
        }
        auto convert_tile = [&](int64_t t, int it) -> bool {
        float v[GROUPS][8];
#pragma unroll
        for (int i = 0; i < GROUPS; ++i) {
            const int gi = ct + 256 * i;
            const int p = gi / CPR, c = gi % CPR;
            const int64_t n = t * kTileP + p;
            if (n < N) {
                load8<XT>(X + n * DX + c * 8, v[i]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) v[i][e] = 0.f;
            }
        }
        // X scale 2^-s (the parameter kernel wrote s before this launch)
        const float xsf = __int_as_float((127 - __ldg(P.xs_exp)) << 23);
#pragma unroll
        for (int i = 0; i < GROUPS; ++i)
#pragma unroll
            for (int e = 0; e < 8; ++e) v[i][e] *= xsf;   // exact: 2^-s
        // lo pieces first (x_lo for fp32 inputs, x2_lo), then hi pieces
        if (it > 0 && !mbar_wait(&bars->xlo_free, (it - 1) & 1, err, abort_flag)) return false;
#pragma unroll
        for (int i = 0; i < GROUPS; ++i) {
            const int gi = ct + 256 * i;
            const int p = gi / CPR, c = gi % CPR;
            const int b = c / 8;
            const uint32_t off = swz128_off(p, c % 8);
            uint32_t wl[4], wsl[4], dummy;
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                const float x0 = v[i][e], x1 = v[i][e + 1];
                split2(x0, x1, dummy, wl[e / 2]);
                split2(x0 * x0, x1 * x1, dummy, wsl[e / 2]);
            }
            if (!XEXACT)
                *reinterpret_cast<uint4 *>(sm + (2 * NB + b) * kBlockBytes + off) =
                    make_uint4(wl[0], wl[1], wl[2], wl[3]);
            *reinterpret_cast<uint4 *>(sm + (3 * NB + b) * kBlockBytes + off) =
                make_uint4(wsl[0], wsl[1], wsl[2], wsl[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->xlo_full);
        if (it > 0 && !mbar_wait(&bars->xhi_free, (it - 1) & 1, err, abort_flag)) return false;
#pragma unroll
        for (int i = 0; i < GROUPS; ++i) {
            const int gi = ct + 256 * i;
            const int p = gi / CPR, c = gi % CPR;
            const int b = c / 8;
            const uint32_t off = swz128_off(p, c % 8);
            uint32_t wh[4], wsh[4], dummy;
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                const float x0 = v[i][e], x1 = v[i][e + 1];
                split2(x0, x1, wh[e / 2], dummy);
                split2(x0 * x0, x1 * x1, wsh[e / 2], dummy);
            }
            *reinterpret_cast<uint4 *>(sm + (0 * NB + b) * kBlockBytes + off) =
                make_uint4(wh[0], wh[1], wh[2], wh[3]);
            *reinterpret_cast<uint4 *>(sm + (1 * NB + b) * kBlockBytes + off) =
                make_uint4(wsh[0], wsh[1], wsh[2], wsh[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->xhi_full);
            return true;
        };
        int it = 0;
        bool live = t_begin >= t_end || convert_tile(t_begin, 0);
        // sweep 1 converts the next tile before the softmax of the last two
        // chunks (its X pieces are released after the last chunk's MMAs; the
        // MMAs of chunk c wait for the softmax of chunk c-2)
        const int conv_at = nchunks >= 2 ? nchunks - 2 : 0;
        for (int64_t t = t_begin; t < t_end && live; t += t_step, ++it) {
            const int64_t n = t * kTileP + p;
            const bool valid = n < N;
            const bool has_next = t + t_step < t_end;
            if (sweep1(MODE)) {
                float m = -INFINITY, l = 0.f;             // in log2 units
                // soft assignment: this thread's best kTopMax (score, id) of
                // its half, descending, ties to the lower component index
                float ts[kTopMax];
                int ti[kTopMax];
#pragma unroll
                for (int j = 0; j < kTopMax; ++j) { ts[j] = -INFINITY; ti[j] = -1; }
                bool ok = true;
                for (int c = 0; c < nchunks; ++c, ++q) {
                    if (c == conv_at && has_next && !convert_tile(t + t_step, it + 1)) { ok = false; break; }
                    const uint32_t buf = q & 1;
                    if (!mbar_wait(&bars->sfull[buf], (q >> 1) & 1, err, abort_flag)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll 1
                    for (int cc = 0; cc < 4; ++cc) {
                        uint32_t r[32];
                        const int col = h * 128 + cc * 32;
                        const int kb = c * kChunk1 + col;
                        tmem_ld32(tmem + lane_base + buf * C + col, r);
                        tmem_ld_wait();
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
                            for (int i = 0; i < 32; ++i) s += ex2_approx(y[i] - nm);
                            l = l * exp2f(m - nm) + s;
                            m = nm;
                        }
                        if constexpr (MODE == kAssign) {
                            // components kb + i in increasing order: a later
                            // equal score never displaces an earlier one
                            if (cm > ts[kTopMax - 1]) {
#pragma unroll
                                for (int i = 0; i < 32; ++i)
                                    if (y[i] > ts[kTopMax - 1]) topr_insert(ts, ti, y[i], kb + i);
                            }
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->sfree[buf]);
                }
                if (!ok) break;
                // merge the two component halves of each point row (the
                // second half first takes in the direct-form components)
                if (h == 1) {
                    if (valid && __ldg(P.dcount) > 0) merge_direct(m, l, __ldg(P.dmf + n));
                    mlx[2 * p] = m;
                    mlx[2 * p + 1] = l;
                }
                if (!reader_sync()) break;
                if (h == 0) {
                    const float m2 = mlx[2 * p], l2 = mlx[2 * p + 1];
                    float mm = fmaxf(m, m2);
                    float ll = 0.f;
                    if (mm != -INFINITY) ll = l * exp2f(m - mm) + l2 * exp2f(m2 - mm);
                    const float lse = (mm + log2f(ll)) * 0.69314718055994531f;
                    if (valid) {
                        if (!(mm > -INFINITY)) set_error(err, GMM_ERR_NONFINITE);
                        lse_out[n] = lse;
                        if (loglik) loglik[n] = lse;
                    }
                    double ds = valid ? (double)lse : 0.0;
#pragma unroll
                    for (int o = 16; o; o >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, o);
                    if (lane == 0) llw[qd] = ds;
                }
                if (!reader_sync()) break;
                if (h == 0 && p == 0) ll_part[t] = (llw[0] + llw[1]) + (llw[2] + llw[3]);
                if constexpr (MODE == kAssign) {
                    // the second half's list joins the first's, one entry per
                    // round through the (m, l) exchange buffer (free again)
                    bool okx = true;
#pragma unroll 1
                    for (int j = 0; j < kTopMax && okx; ++j) {
                        if (h == 1) {
                            mlx[2 * p] = ts[j];
                            mlx[2 * p + 1] = __int_as_float(ti[j]);
                        }
                        okx = reader_sync();
                        if (okx && h == 0) {
                            const float y2 = mlx[2 * p];
                            if (y2 > ts[kTopMax - 1] || (y2 == ts[kTopMax - 1] && y2 > -INFINITY))
                                topr_insert(ts, ti, y2, __float_as_int(mlx[2 * p + 1]));
                        }
                        okx = okx && reader_sync();
                    }
                    if (!okx) break;
                    if (h == 0 && valid) {
                        // direct-form components, from their stored scores
                        const int nd = __ldg(P.dcount);
                        for (int sl = 0; sl < nd; ++sl) {
                            const float y2 = __ldg(A.dscore + (size_t)sl * N + n);
                            if (y2 > ts[kTopMax - 1] || (y2 == ts[kTopMax - 1] && y2 > -INFINITY))
                                topr_insert(ts, ti, y2, __ldg(A.dlist + sl));
                        }
                        // r_nk = 2^(y - l_n); l_n in log2 units
                        const float lse2 = lse_out[n] * kLog2e;
#pragma unroll
                        for (int j = 0; j < kTopMax; ++j) {
                            if (j < A.R) {
                                const float r = ti[j] >= 0 ? exp2f(ts[j] - lse2) : 0.f;
                                const bool keep = ti[j] >= 0 && r >= A.tau;
                                A.ids[n * A.R + j] = keep ? ti[j] : -1;
                                A.resp[n * A.R + j] = keep ? r : 0.f;
                            }
                        }
                    }
                }
            } else {
                const float lse_pref = (MODE == kStats && valid) ? lse_in[n] : 0.f;
                if (!mbar_wait(&bars->sfull[0], it & 1, err, abort_flag)) break;
                tc_fence_after();
                float lse2;   // l_n in log2 units
                if (MODE == kSingle) {
                    float m = -INFINITY, l = 0.f;
                    for (int cc = 0; cc < 2; ++cc) {
                        const int col = h * 64 + cc * 32;
                        uint32_t r[32];
                        tmem_ld32(tmem + lane_base + col, r);
                        tmem_ld_wait();
                        float y[32], cm = -INFINITY;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            y[i] = fmaf(__uint_as_float(r[i]), cA[col + i], cB[col + i]);
                            cm = fmaxf(cm, y[i]);
                        }
                        const float nm = fmaxf(m, cm);
                        if (nm != -INFINITY) {
                            float s = 0.f;
#pragma unroll
                            for (int i = 0; i < 32; ++i) s += ex2_approx(y[i] - nm);
                            l = l * exp2f(m - nm) + s;
                            m = nm;
                        }
                    }
                    mlx[(h * kSlice + p) * 2] = m;
                    mlx[(h * kSlice + p) * 2 + 1] = l;
                    if (!reader_sync()) break;
                    const float m2 = mlx[((1 - h) * kSlice + p) * 2];
                    const float l2 = mlx[((1 - h) * kSlice + p) * 2 + 1];
                    // combine in a fixed order (half 0 first) so both halves agree bitwise
                    const float ma = h == 0 ? m : m2, la = h == 0 ? l : l2;
                    const float mb = h == 0 ? m2 : m, lb = h == 0 ? l2 : l;
                    float mm = fmaxf(ma, mb);
                    float ll = 0.f;
                    if (mm != -INFINITY) ll = la * exp2f(ma - mm) + lb * exp2f(mb - mm);
                    if (valid && __ldg(P.dcount) > 0) merge_direct(mm, ll, __ldg(P.dmf + n));
                    lse2 = mm + log2f(ll);
                    if (h == 0) {
                        const float lse = lse2 * 0.69314718055994531f;
                        if (valid) {
                            if (!(mm > -INFINITY)) set_error(err, GMM_ERR_NONFINITE);
                            lse_out[n] = lse;
                            if (loglik) loglik[n] = lse;
                        }
                        double ds = valid ? (double)lse : 0.0;
#pragma unroll
                        for (int o = 16; o; o >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, o);
                        if (lane == 0) llw[qd] = ds;
                    }
                } else {
                    lse2 = lse_pref * kLog2e;
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
                // Pass A: per component of this half, max over the
                // quadrant's 32 points of ceil(log2 r_nk).
                for (int cc = 0; cc < 2; ++cc) {
                    const int col = h * 64 + cc * 32;
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_base + col, r);
                    tmem_ld_wait();
                    int mine = -250;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float e = fmaf(__uint_as_float(r[i]), cA[col + i], cB[col + i]) - lse2;
                        const int ce = (int)ceilf(fmaxf(e, -250.f));
                        const int mx = __reduce_max_sync(0xffffffffu, ce);
                        if (lane == i) mine = mx;
                    }
                    tmax[qd * kSlice + col + lane] = mine;
                }
                if (!reader_sync()) break;
                if (MODE == kSingle && h == 0 && p == 0)
                    ll_part[t] = (llw[0] + llw[1]) + (llw[2] + llw[3]);
                if (h == 0) {
                    // thread p owns component p's scale and TMEM statistics row
                    const int tm = max(max(tmax[p], tmax[kSlice + p]),
                                       max(tmax[2 * kSlice + p], tmax[3 * kSlice + p]));
                    const int s_old = (it == 0) ? kSigInit : sig[p];
                    const int s_new = min(s_old, 15 - tm);
                    sig[p] = s_new;
                    const int delta = s_new - s_old;
                    if (it > 0 && it % kFlushTiles == 0) {
                        // bound the fp32 accumulation chain: the statistics
                        // are idle (the previous M-step completed before this
                        // tile's scores did); move them into the fp64 partial
                        const double sc = exp2i_d(-s_old);
                        double *out = partial + (size_t)blockIdx.y * ((size_t)K * (1 + 2 * (size_t)DX));
#pragma unroll 1
                        for (int cc = -1; cc < 2 * D / 16; ++cc)
                            flush_stats_chunk<D, DX>(t_s0 + lane_base, t_st + lane_base, cc, out, K,
                                                     comp0 + p, sc, nflush > 0, true, __ldg(P.xs_exp));
                        tmem_st_wait();
                        ++nflush;
                    } else if (it > 0 && __any_sync(0xffffffffu, delta < 0)) {
                        // the previous M-step completed before this tile's
                        // scores did, so the statistics are idle: rescale
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
                    tc_fence_before();
                }
                if (!reader_sync()) break;
                tc_fence_after();
                // Pass B: r'_nk = 2^(y_nk - l_n + sig_k) -> r_hi / r_lo of this
                // half's 64-component block (MN-major, SWIZZLE_128B)
                uint8_t *rhi = sm + S::RING + h * kBlockBytes;
                uint8_t *rlo = rhi + 2 * kBlockBytes;
                for (int cc = 0; cc < 2; ++cc) {
                    const int col = h * 64 + cc * 32;
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_base + col, r);
                    tmem_ld_wait();
                    uint32_t ph[16], pl[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        const float y0 = fmaf(__uint_as_float(r[i]), cA[col + i], cB[col + i]) -
                                         lse2 + (float)sig[col + i];
                        const float y1 = fmaf(__uint_as_float(r[i + 1]), cA[col + i + 1],
                                              cB[col + i + 1]) - lse2 + (float)sig[col + i + 1];
                        split2(ex2_approx(y0), ex2_approx(y1), ph[i / 2], pl[i / 2]);
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t off = swz128_off(p, cc * 4 + j);
                        *reinterpret_cast<uint4 *>(rhi + off) =
                            make_uint4(ph[4 * j], ph[4 * j + 1], ph[4 * j + 2], ph[4 * j + 3]);
                        *reinterpret_cast<uint4 *>(rlo + off) =
                            make_uint4(pl[4 * j], pl[4 * j + 1], pl[4 * j + 2], pl[4 * j + 3]);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->rq[qd]);
                if (has_next && !convert_tile(t + t_step, it + 1)) break;
            }
        }
        if (!sweep1(MODE) && h == 0) {
            // drain the slice's statistics: lane = component row
            if (mbar_wait(&bars->done, 0, err, abort_flag)) {
                tc_fence_after();
                // (a CTA without tiles never ran an M-step: it writes zeros)
                const double sc = (t_begin < t_end) ? exp2i_d(-sig[p]) : 0.0;
                double *out = partial + (size_t)blockIdx.y * ((size_t)K * (1 + 2 * (size_t)DX));
#pragma unroll 1
                for (int cc = -1; cc < 2 * D / 16; ++cc)
                    flush_stats_chunk<D, DX>(t_s0 + lane_base, t_st + lane_base, cc, out, K,
                                             comp0 + p, sc, nflush > 0, false, __ldg(P.xs_exp));
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
    // d = 32 runs padded to one 64-feature block (the direct-form kernels
    // take features 32 at a time)
    return (d == 32 || d == 64 || d == 128) && K >= 1 && K <= 4096 * 4;
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

// The tensor-core region of the workspace (byte offsets): parameter image,
// a_k, b_k, then the direct-form bookkeeping, the [cap x C] scores and the
// per-point (max, sum) of the direct-form components for a chunk of C
// points.
struct TcLayout {
    size_t ak, bk, dflag, dlist, dscore, dmf, dpart, xmax, skpart, total;
    int cap;
};

// A step over N points runs as a sequence of point chunks, each the whole
// launch sequence on its rows, so that the direct-form scores are held for
// one chunk at a time (the method's point is that nothing of size N x K is
// kept; Flash-GMM abstract).  The score block may take as many bytes as X
// at 16 bits per element, clamped to [512 MiB, 4 GiB]: no chunking while it
// is no larger than the data (every chunk repeats the per-call launches and
// a persistent kernel's ramp and tail), and a bound of 4 GiB past that
// however large N is.  A chunk is a whole number of waves of 128-point
// tiles (kMaxRanges tiles) unless it is all of N, and the chunks are of
// equal size but the last.
constexpr size_t kDirBlockMin = (size_t)512 << 20;
constexpr size_t kDirBlockMax = (size_t)4 << 30;
constexpr int64_t kChunkWave = (int64_t)kTileP * kMaxRanges;
int64_t g_chunk_override = 0;   // gmm_set_point_chunk; 0 = automatic

// Points per chunk when nothing overrides it; the workspace is laid out for
// this many.
int64_t tc_block_points(int64_t N, int d, int K) {
    if (N < 1) return 1;
    const size_t per = (size_t)direct_slots(K) * 4;
    size_t budget = (size_t)N * (size_t)d * 2;
    if (budget < kDirBlockMin) budget = kDirBlockMin;
    if (budget > kDirBlockMax) budget = kDirBlockMax;
    if (per * (size_t)N <= budget) return N;
    int64_t cmax = (int64_t)(budget / per) / kChunkWave * kChunkWave;
    if (cmax < kChunkWave) cmax = kChunkWave;
    const int64_t nch = (N + cmax - 1) / cmax;
    const int64_t c = ((N + nch - 1) / nch + kChunkWave - 1) / kChunkWave * kChunkWave;
    return c < cmax ? c : cmax;
}

// Shapes the small-mixture kernel takes: 16-bit data, d = 32, K <= 32, one
// sweep.  Its fp64 partial rows: one CTA per SM at most, 4 x 32 rows of
// kSmallCols columns.
bool smallk_shape(int d, int K) { return d == kSmallD && K <= 32; }
size_t smallk_part_bytes(int d, int K) {
    return smallk_shape(d, K) ? (size_t)kMaxRanges * kSmallF * (4 * 32) * 8 : 0;
}

TcLayout tc_layout(int64_t N, int d, int K, int Kp) {
    TcLayout L;
    L.cap = direct_slots(K);
    const size_t n = (size_t)tc_block_points(N, d, K);
    size_t o = align_up(img_bytes(Kp, (d + 63) / 64));
    L.ak = o;     o += align_up((size_t)Kp * 4);
    L.bk = o;     o += align_up((size_t)Kp * 4);
    L.dflag = o;  o += align_up((size_t)Kp * 4);
    L.dlist = o;  o += align_up((size_t)(kDirectMax + 1) * 4);
    L.dscore = o; o += align_up((size_t)L.cap * n * 4);
    L.dmf = o;    o += align_up(n * 8);
    L.dpart = o;  o += align_up((size_t)L.cap * kDirRanges * (1 + 2 * (size_t)d) * 8);
    L.xmax = o;   o += align_up(8);   // max |x| bits, X scale exponent
    L.skpart = o; o += align_up(smallk_part_bytes(d, K));
    L.total = o;
    return L;
}

}  // namespace

int64_t gmm_tc_chunk_points(int64_t N, int d, int K) {
    const int64_t c = tc_block_points(N, d, K);
    if (g_chunk_override <= 0) return c;
    const int64_t o = (g_chunk_override + kTileP - 1) / kTileP * kTileP;
    return o < c ? o : c;
}

void gmm_tc_set_chunk_override(int64_t points) { g_chunk_override = points > 0 ? points : 0; }

bool gmm_tc_supported(gmm_dtype dt, int64_t N, int d, int K, uint32_t flags) {
    (void)N;
    (void)flags;
    return tc_shape_ok(dt, d, K);
}

int gmm_tc_regime(gmm_dtype dt, int64_t N, int d, int K, uint32_t flags) {
    (void)dt; (void)N; (void)d;
    if (K > kClu * kSlice || (flags & GMM_FLAG_FORCE_TWO_SWEEP)) return 2;
    return 1;
}

bool gmm_tc_runs_fused(gmm_dtype dt, int64_t N, int d, int K, uint32_t flags) {
    const bool two = gmm_tc_regime(dt, N, d, K, flags) == 2;
    return two || tc_kp(K) != kClu * kSlice;
}

size_t gmm_tc_ws_bytes(int64_t N, int d, int K) {
    if (!tc_shape_ok(GMM_F32, d, K)) return 0;
    int Kp = tc_kp(K);
    if (Kp < kChunk1) Kp = kChunk1;   // the two-sweep flag pads to a 256 multiple
    return tc_layout(N, d, K, Kp).total;
}

int64_t gmm_tc_max_partials(int64_t N, int d, int K) {
    (void)d;
    const int64_t ntiles = (N + kTileP - 1) / kTileP;   // every range holds at least a tile
    int64_t rows = ntiles < kMaxRanges ? ntiles : kMaxRanges;
    if (K > kClu * kSlice) {   // always two sweeps: one row per point range of a slice
        int Kp = tc_kp(K);
        if (Kp < kChunk1) Kp = kChunk1;
        int64_t r = kMaxRanges / (Kp / kSlice);
        if (r < 1) r = 1;
        if (r < rows) rows = r;
    }
    return rows;
}

int64_t gmm_tc_max_ll(int64_t N, int d, int K) {
    (void)d; (void)K;
    const int64_t tiles = (N + kTileP - 1) / kTileP;
    return tiles > 12 * kMaxRanges ? tiles : 12 * kMaxRanges;   // (small-K kernel: 12 per CTA)
}

// max |x| into *xmax (cleared first): one read of X, grid-stride, two
// blocks per SM.
template <typename XT>
static cudaError_t launch_direct(unsigned blocks, const XT *X, int64_t N, int d,
                                 const float *means, const float *vars, const float *logw,
                                 const int *dlist, const int *dcount, float *dscore,
                                 float2 *dmf, uint32_t *xmax, cudaStream_t s) {
    auto kern = gmm_tc_direct_scores_kernel<XT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kDirSmem);
    if (e != cudaSuccess) return e;
    static int per_sm = 0;   // resident blocks per SM, asked once
    if (per_sm == 0) {
        int nb = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kDirThreads, kDirSmem) != cudaSuccess ||
            nb < 1)
            nb = 1;
        per_sm = nb;
    }
    const unsigned cap = (unsigned)(per_sm * tc_sm_count());
    if (blocks > cap) blocks = cap;
    kern<<<blocks, kDirThreads, kDirSmem, s>>>(X, N, d, means, vars, logw, dlist, dcount, dscore,
                                               dmf, xmax);
    return cudaGetLastError();
}

template <int NB, typename XT, int MODE, int DX>
static cudaError_t launch_fused(dim3 grid, const XT *X, int64_t N, int K, const TcParams &P,
                                const GmmWs &w, float *loglik, int64_t tiles_per_range,
                                cudaStream_t s, const AssignOut &A = AssignOut{}) {
    auto kern = gmm_tc_fused_kernel<NB, XT, MODE, DX>;
    const int smem = Smem<NB, MODE>::TOTAL;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, s>>>(X, N, K, P, w.lse, w.lse, loglik, w.ll_part, w.partial64,
                                      tiles_per_range, w.err, A);
    return cudaGetLastError();
}

// Single sweep over a cluster of kClu CTAs (128 < K <= 256).  The grid is
// one wave of clusters: as many as fit on the device at once (a cluster
// needs kClu SMs of one GPC), each taking a contiguous range of tiles.
template <int NB, typename XT, int DX>
static cudaError_t launch_cluster(const XT *X, int64_t N, int K, const TcParams &P,
                                  const GmmWs &w, float *loglik, int *num_partials,
                                  int64_t *num_ll, cudaStream_t s) {
    auto kern = gmm_tc_cluster_kernel<NB, XT, DX>;
    const int smem = SmemC<NB>::TOTAL;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kClu;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreadsC);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    static int max_clusters = 0;   // per process: one device model
    if (max_clusters <= 0) {
        cfg.gridDim = dim3(kClu, kMaxRanges / kClu);
        int nc = 0;
        if (cudaOccupancyMaxActiveClusters(&nc, kern, &cfg) != cudaSuccess || nc < 1) {
            (void)cudaGetLastError();
            nc = tc_sm_count() / kClu;
        }
        max_clusters = nc < kMaxRanges ? nc : kMaxRanges;
    }
    const int64_t ntiles = (N + kTileP - 1) / kTileP;
    int ranges = max_clusters;
    if (ranges > ntiles) ranges = (int)ntiles;
    const int64_t tpr = (ntiles + ranges - 1) / ranges;
    ranges = (int)((ntiles + tpr - 1) / tpr);
    *num_partials = ranges;
    *num_ll = ntiles;
    cfg.gridDim = dim3(kClu, ranges);
    timer_begin(s);
    e = cudaLaunchKernelEx(&cfg, kern, X, N, K, P, w.lse, loglik, w.ll_part, w.partial64, tpr,
                           w.err);
    note_launches(1);
    timer_end(s);
    return e;
}

template <int NB, typename XT, int DX>
static cudaError_t launch_tc_t(const XT *X, int64_t N, int K, const TcParams &P, const GmmWs &w,
                               float *loglik, bool two_sweep, int *num_partials, int64_t *num_ll,
                               cudaStream_t s) {
    if (!two_sweep && P.Kp == kClu * kSlice)
        return launch_cluster<NB, XT, DX>(X, N, K, P, w, loglik, num_partials, num_ll, s);
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
        e = launch_fused<NB, XT, kLse, DX>(dim3(g1), X, N, K, P, w, loglik, 0, s);
        if (e != cudaSuccess) return e;
        {
            auto kern = gmm_tc_stats_kernel<NB, XT, DX>;
            const int smem = SmemT<NB>::TOTAL;
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e != cudaSuccess) return e;
            kern<<<dim3(slices, ranges), kThreads, smem, s>>>(X, N, K, P, w.lse, w.partial64, tpr,
                                                             w.err);
            e = cudaGetLastError();
        }
        note_launches(2);
    } else {
        e = launch_fused<NB, XT, kSingle, DX>(dim3(1, ranges), X, N, K, P, w, loglik, tpr, s);
        note_launches(1);
    }
    timer_end(s);
    return e;
}

// Everything before the fused kernels: max|x| and the X scale, the
// parameter pieces, the direct-form list and the direct-form scores.  X and
// N are one chunk's rows; n_ws is the N the workspace was sized for.  The
// conditioning and the list depend on the parameters alone: a later chunk
// of the same call (later = true) keeps them.
static cudaError_t tc_prepare(const void *X, gmm_dtype dt, int64_t N, int64_t n_ws, int d, int K,
                              const float *means, const float *vars, const float *logw,
                              const GmmWs &w, int Kp, uint32_t flags, bool later, TcParams *P,
                              int **dlist_out, float **dscore_out, cudaStream_t s) {
    // offsets as sized by gmm_tc_ws_bytes (Kp padded to a 256 multiple)
    const TcLayout L = tc_layout(n_ws, d, K, Kp < kChunk1 ? kChunk1 : Kp);
    char *base = (char *)w.tc;
    uint8_t *img = (uint8_t *)base;
    float *ak = (float *)(base + L.ak), *bk = (float *)(base + L.bk);
    int *dflag = (int *)(base + L.dflag);
    int *dlist = (int *)(base + L.dlist), *dcount = dlist + kDirectMax;
    float *dscore = (float *)(base + L.dscore);
    float2 *dmf = (float2 *)(base + L.dmf);
    uint32_t *xmax = (uint32_t *)(base + L.xmax);
    int *xs_exp = (int *)(base + L.xmax + 4);
    // conditioning and the direct-form list (independent of the data), then
    // one pass over X for the listed components' scores and max|x|, then the
    // parameter image at the X scale that max|x| fixes
    cudaError_t e = cudaMemsetAsync(xmax, 0, 4, s);
    if (e != cudaSuccess) return e;
    if (!later) {
        gmm_tc_cond_kernel<<<(Kp * 32 + 255) / 256, 256, 0, s>>>(means, vars, logw, K, d, Kp, bk,
                                                                 dflag, w.err);
        gmm_tc_direct_list_kernel<<<1, 1024, 0, s>>>(dflag, Kp, L.cap, bk, dlist, dcount, w.err);
        note_launches(2);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    {
        // one 32-point tile per warp, capped at one wave
        int64_t blocks = ((N + kDirPts - 1) / kDirPts + kDirWarps - 1) / kDirWarps;
        if (blocks > (1 << 30)) blocks = 1 << 30;
        if (blocks < 1) blocks = 1;
        if (dt == GMM_F32)
            e = launch_direct<float>((unsigned)blocks, (const float *)X, N, d, means, vars, logw,
                                     dlist, dcount, dscore, dmf, xmax, s);
        else if (dt == GMM_BF16)
            e = launch_direct<__nv_bfloat16>((unsigned)blocks, (const __nv_bfloat16 *)X, N, d,
                                             means, vars, logw, dlist, dcount, dscore, dmf, xmax, s);
        else
            e = launch_direct<__half>((unsigned)blocks, (const __half *)X, N, d, means, vars,
                                      logw, dlist, dcount, dscore, dmf, xmax, s);
        note_launches(1);
        if (e != cudaSuccess) return e;
    }
    gmm_tc_params_kernel<<<(Kp * 32 + 255) / 256, 256, 0, s>>>(means, vars, K, d, Kp, xmax, xs_exp,
                                                               img, ak, dflag, w.err);
    note_launches(1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // the stalled stage lies inside the first tile's E-step program
    *P = TcParams{img, ak, bk, Kp, dmf, dcount, xs_exp, (flags & GMM_FLAG_TEST_STALL) ? 3 : -1};
    if (dlist_out) *dlist_out = dlist;
    if (dscore_out) *dscore_out = dscore;
    return cudaSuccess;
}

// The small-mixture kernel (16-bit data, d = 32, K <= 32) and the fixed-order
// reduction of its partial rows straight into `stats` (*num_partials = -1:
// nothing left for the caller's reduction; accumulate: add into `stats`).
template <typename XT>
static cudaError_t launch_smallk(const XT *X, int64_t N, int K, const TcParams &P,
                                 const GmmWs &w, float *loglik, double *part, double *stats,
                                 bool accumulate, int *num_partials, int64_t *num_ll,
                                 cudaStream_t s) {
    const int64_t ntiles = (N + kTileP - 1) / kTileP;
    int grid = tc_sm_count();
    if (grid > kMaxRanges) grid = kMaxRanges;
    if (grid > ntiles) grid = (int)ntiles;
    cudaError_t e;
    timer_begin(s);
    if (K <= 16) {
        auto kern = gmm_tc_smallk_kernel<XT, 16>;
        const int smem = SmemS<16>::TOTAL;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, small_threads(16), smem, s>>>(X, N, P, w.lse, loglik, w.ll_part, part, w.err);
        timer_end(s);
        gmm_tc_smallk_reduce_kernel<16><<<(K * (1 + 2 * kSmallD) + 7) / 8, 256, 0, s>>>(
            part, grid, K, stats, accumulate);
    } else {
        auto kern = gmm_tc_smallk_kernel<XT, 32>;
        const int smem = SmemS<32>::TOTAL;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, small_threads(32), smem, s>>>(X, N, P, w.lse, loglik, w.ll_part, part, w.err);
        timer_end(s);
        gmm_tc_smallk_reduce_kernel<32><<<(K * (1 + 2 * kSmallD) + 7) / 8, 256, 0, s>>>(
            part, grid, K, stats, accumulate);
    }
    note_launches(2);
    *num_partials = -1;
    *num_ll = 4 * small_groups(K <= 16 ? 16 : 32) * (int64_t)grid;   // one total per worker warp
    return cudaGetLastError();
}

cudaError_t launch_gmm_tc(const void *X, gmm_dtype dt, int64_t N, int64_t n_ws, int d, int K,
                          const float *means, const float *vars, const float *logw,
                          const GmmWs &w, float *loglik, uint32_t flags, int *num_partials,
                          int64_t *num_ll, double *stats, bool accumulate, cudaStream_t s) {
    if (!tc_shape_ok(dt, d, K)) return cudaErrorNotSupported;
    const bool two = gmm_tc_regime(dt, N, d, K, flags) == 2;
    int Kp = tc_kp(K);
    if (two && Kp < kChunk1) Kp = kChunk1;
    TcParams P;
    cudaError_t e = tc_prepare(X, dt, N, n_ws, d, K, means, vars, logw, w, Kp, flags, accumulate,
                               &P, nullptr, nullptr, s);
    if (e != cudaSuccess) return e;
    if (dt != GMM_F32 && smallk_shape(d, K) && !two && !(flags & GMM_FLAG_TEST_STALL)) {
        const TcLayout L = tc_layout(n_ws, d, K, Kp < kChunk1 ? kChunk1 : Kp);
        double *part = (double *)((char *)w.tc + L.skpart);
        if (dt == GMM_BF16)
            return launch_smallk<__nv_bfloat16>((const __nv_bfloat16 *)X, N, K, P, w, loglik,
                                                part, stats, accumulate, num_partials, num_ll, s);
        return launch_smallk<__half>((const __half *)X, N, K, P, w, loglik, part, stats,
                                     accumulate, num_partials, num_ll, s);
    }
#define GMM_TC_CASE(NBV, DXV, T)                                                               \
    return launch_tc_t<NBV, T, DXV>((const T *)X, N, K, P, w, loglik, two, num_partials, num_ll, s)
#define GMM_TC_DTYPES(NBV, DXV)                                                                \
    do {                                                                                       \
        if (dt == GMM_F32) GMM_TC_CASE(NBV, DXV, float);                                       \
        if (dt == GMM_BF16) GMM_TC_CASE(NBV, DXV, __nv_bfloat16);                              \
        GMM_TC_CASE(NBV, DXV, __half);                                                         \
    } while (0)
    switch (d) {
    case 32: GMM_TC_DTYPES(1, 32);
    case 64: GMM_TC_DTYPES(1, 64);
    default: GMM_TC_DTYPES(2, 128);
    }
#undef GMM_TC_DTYPES
#undef GMM_TC_CASE
}

// Soft assignment on the tensor cores: sweep 1 over 256-component chunks
// with the per-point top-kTopMax selection (kAssign), persistent over the
// point tiles; l_n goes to w.lse (and loglik), the selection to ids / resp.
cudaError_t launch_gmm_tc_assign(const void *X, gmm_dtype dt, int64_t N, int64_t n_ws, int d,
                                 int K, const float *means, const float *vars, const float *logw,
                                 const GmmWs &w, float *loglik, int R, float tau, int32_t *ids,
                                 float *resp, bool later, cudaStream_t s) {
    if (!tc_shape_ok(dt, d, K)) return cudaErrorNotSupported;
    int Kp = tc_kp(K);
    if (Kp < kChunk1) Kp = kChunk1;
    TcParams P;
    int *dlist = nullptr;
    float *dscore = nullptr;
    cudaError_t e = tc_prepare(X, dt, N, n_ws, d, K, means, vars, logw, w, Kp, 0, later, &P, &dlist,
                               &dscore, s);
    if (e != cudaSuccess) return e;
    const AssignOut A{R, tau, ids, resp, dlist, dscore};
    const int64_t ntiles = (N + kTileP - 1) / kTileP;
    int g1 = tc_sm_count();
    if (g1 > ntiles) g1 = (int)ntiles;
    timer_begin(s);
#define GMM_TA_CASE(NBV, DXV, T)                                                               \
    e = launch_fused<NBV, T, kAssign, DXV>(dim3(g1), (const T *)X, N, K, P, w, loglik, 0, s, A)
    if (d == 32) {
        if (dt == GMM_F32) GMM_TA_CASE(1, 32, float);
        else if (dt == GMM_BF16) GMM_TA_CASE(1, 32, __nv_bfloat16);
        else GMM_TA_CASE(1, 32, __half);
    } else if (d == 64) {
        if (dt == GMM_F32) GMM_TA_CASE(1, 64, float);
        else if (dt == GMM_BF16) GMM_TA_CASE(1, 64, __nv_bfloat16);
        else GMM_TA_CASE(1, 64, __half);
    } else {
        if (dt == GMM_F32) GMM_TA_CASE(2, 128, float);
        else if (dt == GMM_BF16) GMM_TA_CASE(2, 128, __nv_bfloat16);
        else GMM_TA_CASE(2, 128, __half);
    }
#undef GMM_TA_CASE
    note_launches(1);
    timer_end(s);
    return e;
}

cudaError_t launch_gmm_tc_direct_stats(const void *X, gmm_dtype dt, int64_t N, int64_t n_ws,
                                       int d, int K, const GmmWs &w, double *stats,
                                       cudaStream_t s) {
    int Kp = tc_kp(K);
    if (Kp < kChunk1) Kp = kChunk1;   // the layout is the same for either regime
    const TcLayout L = tc_layout(n_ws, d, K, Kp);
    const char *base = (const char *)w.tc;
    const int *dlist = (const int *)(base + L.dlist), *dcount = dlist + kDirectMax;
    const float *dscore = (const float *)(base + L.dscore);
    double *dpart = (double *)(base + L.dpart);
    // at most kDirRanges ranges of at least 16384 points: a chunk of a long
    // step writes (and the final kernel reads) few partial rows
    int64_t span = (N + kDirRanges - 1) / kDirRanges;
    if (span < 16384) span = 16384;
    span = (span + 255) / 256 * 256;
    const int nr = (int)((N + span - 1) / span);
    const dim3 grid(L.cap, nr);
    if (dt == GMM_F32)
        gmm_tc_direct_stats_kernel<float><<<grid, 256, 0, s>>>((const float *)X, N, d, span, dcount,
                                                               dscore, w.lse, dpart);
    else if (dt == GMM_BF16)
        gmm_tc_direct_stats_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
            (const __nv_bfloat16 *)X, N, d, span, dcount, dscore, w.lse, dpart);
    else
        gmm_tc_direct_stats_kernel<__half><<<grid, 256, 0, s>>>((const __half *)X, N, d, span,
                                                                dcount, dscore, w.lse, dpart);
    gmm_tc_direct_stats_final<<<L.cap, 256, 0, s>>>(d, K, nr, dlist, dcount, dpart, stats);
    note_launches(2);
    return cudaGetLastError();
}

}  // namespace gmmb
