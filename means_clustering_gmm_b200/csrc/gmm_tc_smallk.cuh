// Single-sweep EM for small mixtures of 16-bit data (K <= 32, d = 32): a
// persistent kernel that streams X at HBM rate.  Included by gmm_tc.cu after
// the shared definitions; not a separate translation unit.
//
// With few components the per-point work is small and the run is bound by
// the one read of X ("Flash-GMM: a memory-efficient kernel for scalable soft
// clustering", abstract: the whole iteration in one pass over the data), so
// the design keeps every unit busy on 128-point tiles:
//   - warp 0 copies raw X tiles (128 rows, contiguous) into a 6-stage ring
//     with 1-D bulk copies;
//   - warps 2.. are NG groups of four (one warp per TMEM lane quadrant;
//     NG = 3 for K <= 16, 2 for K <= 32); group g takes the CTA's tiles i
//     with i % NG == g.  A thread owns one
//     point of the tile: it converts the row into the operand tile
//     [x | x^2_hi | x^2_lo | 1 | 0] (128 features; 16-bit x is exact in
//     fp16), and after the E-step reads the point's scores, forms l_n and the
//     responsibilities and writes them as the M-step's other operand;
//   - warp 1 issues the MMAs, each as soon as its inputs are ready (it polls
//     both queues, so one tile's M-step never waits behind the next tile's
//     E-step):
//       E-step  D_E[pt, 0..2KP) = A[pt, 0..3d) . B_E^T, B_E rows
//               hi: [W1_hi | W2_hi | 0], lo: [W1_lo | W2_lo | W2_hi]: the
//               large products and the corrections land in separate
//               accumulators (no truncation of the small terms at the large
//               terms' magnitude); s_k = (hi_k + lo_k) a_k + b_k;
//       M-step  D_M[f, row] += A[pt, f]^T . R[pt, row] over the tile's
//               points: lanes are the 128 operand features (S1 from x, S2
//               from x^2_hi + x^2_lo, S0 from the ones), columns the 4 KP
//               rows [r_big hi | r_big lo | r_small hi | r_small lo].
//     r_nk >= 2^-23 enters as r 2^14 (big), smaller ones as r 2^38 (small),
//     each split into an fp16 hi/lo pair, so every responsibility keeps 22
//     bits whatever the component's mass, with no per-component running
//     scale.
//   - every kSmallFlush tiles (and after the last) the group that ran the
//     tile moves D_M into the CTA's fp64 partial rows (single writer per
//     element: plain store first, reductions after) while the issuer holds
//     the next M-step; this bounds the truncating fp32 accumulation chain as
//     in the other kernels.
// All waits are bounded (tc::mbar_wait, or the issuer's progress timer); an
// abort drains the bulk copies and MMAs this CTA has in flight before TMEM
// is freed.

namespace {

constexpr int kSmallD = 32;              // features
constexpr int kSmallStages = 6;          // raw X ring
// worker groups (tiles in flight): three when K <= 16 (124 registers a
// thread fit 14 warps), two when K <= 32
__host__ __device__ constexpr int small_groups(int KP) { return KP <= 16 ? 3 : 2; }
__host__ __device__ constexpr int small_threads(int KP) { return 64 + 128 * small_groups(KP); }
constexpr int kSmallFlush = 64;          // tiles between statistics flushes
constexpr int kSmallF = 128;             // operand features: [x | x2_hi | x2_lo | ones | 0]

template <int KP>
struct SmemS {
    static constexpr int NG = small_groups(KP);
    static constexpr int XRAW = kTileP * kSmallD * 2;            // 8 KB raw tile
    static constexpr int ATILE = 2 * kBlockBytes;                // 128 features, 32 KB
    static constexpr int RTILE = ((4 * KP + 63) / 64) * kBlockBytes;   // 4KP rows, MN-major
    static constexpr int BE = 2 * (2 * KP) * 128;                // E-step B: 2 blocks x 2KP rows
    static constexpr int A0 = 0;                                 // operand tiles (NG groups)
    static constexpr int R0 = A0 + NG * ATILE;                   // R tiles (NG groups)
    static constexpr int X0 = R0 + NG * RTILE;                   // raw ring
    static constexpr int B0 = X0 + kSmallStages * XRAW;          // B_E
    static constexpr int C0 = B0 + BE;                           // a_k, b_k
    static constexpr int BARS = C0 + 2 * KP * 4;
    static constexpr int TOTAL = BARS + 512 + 1024;              // barriers, misc, alignment
    static_assert(TOTAL <= 232448, "shared memory budget");
};

struct BarsS {
    uint64_t xfull[kSmallStages], xempty[kSmallStages];
    uint64_t afull[3], sfull[3], sfree[3], rfull[3], mfree[3];
    uint64_t flushgo, flushdone, done;
};

}  // namespace

template <typename XT, int KP>
__global__ void __launch_bounds__(small_threads(KP), 1)
gmm_tc_smallk_kernel(const XT *__restrict__ X, int64_t N, TcParams P, float *__restrict__ lse_out,
                     float *__restrict__ loglik, double *__restrict__ ll_part,
                     double *__restrict__ partial, int *err) {
    using S = SmemS<KP>;
    constexpr int D = kSmallD;
    constexpr int NE = 2 * KP;                  // E-step N (hi | lo)
    constexpr int NM = 4 * KP;                  // M-step N (the four R row groups)
    constexpr int KE = 3 * D / 16;              // E-step K steps (6)
    constexpr int NG = S::NG;                   // worker groups
    constexpr int NT = small_threads(KP);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    BarsS *bars = reinterpret_cast<BarsS *>(sm + S::BARS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S::BARS + 256);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + S::BARS + 260);
    float *cA = reinterpret_cast<float *>(sm + S::C0);
    float *cB = cA + KP;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t ntiles = (N + kTileP - 1) / kTileP;
    // this CTA's tiles: blockIdx.x, blockIdx.x + gridDim.x, ...
    const int64_t my_tiles = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (tid == 0) {
        for (int s = 0; s < kSmallStages; ++s) {
            mbar_init(&bars->xfull[s], 1);
            mbar_init(&bars->xempty[s], 4);
        }
        for (int g = 0; g < NG; ++g) {
            mbar_init(&bars->afull[g], 4);
            mbar_init(&bars->sfull[g], 1);
            mbar_init(&bars->sfree[g], 4);
            mbar_init(&bars->rfull[g], 4);
            mbar_init(&bars->mfree[g], 1);
        }
        mbar_init(&bars->flushgo, 1);
        mbar_init(&bars->flushdone, 4);
        mbar_init(&bars->done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // E-step B image: rows 0..KP-1 hi [W1_hi | W2_hi | 0], rows KP..2KP-1 lo
    // [W1_lo | W2_lo | W2_hi], features in two 64-feature SWIZZLE_128B blocks
    for (int i = tid; i < NE * 3 * D; i += NT) {
        const int r = i / (3 * D), f = i % (3 * D);
        const int k = r % KP;
        const bool lo = r >= KP;
        const int part = f / D, j = f % D;   // 0: x, 1: x2_hi, 2: x2_lo
        int piece = -1;
        if (part == 0) piece = lo ? 1 : 0;
        else if (part == 1) piece = lo ? 3 : 2;
        else if (lo) piece = 2;
        __half v = __float2half_rn(0.f);
        if (piece >= 0)
            v = *reinterpret_cast<const __half *>(P.img + img_elem(piece, 0, k, j, 1, P.Kp));
        *reinterpret_cast<__half *>(sm + S::B0 + (f / 64) * (NE * 128) +
                                    swz128_off(r, (f % 64) / 8) + (f % 8) * 2) = v;
    }
    for (int i = tid; i < KP; i += NT) {
        cA[i] = P.ak[i];
        cB[i] = P.bk[i];
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
    // TMEM columns: E-step scores of group g at g * 64, M-step statistics after
    const uint32_t t_m = tmem + NG * 64;

    if (warp == 0) {
        // ===================== raw X tiles -> ring (1-D bulk copies)
        if (lane == 0) {
            int64_t i = 0;
            for (; i < my_tiles && !*abort_flag; ++i) {
                const int st = (int)(i % kSmallStages);
                if (!mbar_wait(&bars->xempty[st], (uint32_t)(((i / kSmallStages) & 1) ^ 1), err,
                               abort_flag))
                    break;
                const int64_t t = blockIdx.x + i * gridDim.x;
                const int64_t rows = min((int64_t)kTileP, N - t * kTileP);
                const uint32_t bytes = (uint32_t)(rows * D * (int64_t)sizeof(XT));
                mbar_arrive_expect_tx(&bars->xfull[st], bytes);
                bulk_g2s(sm + S::X0 + st * S::XRAW, X + t * kTileP * D, bytes, &bars->xfull[st]);
            }
            // no bulk copy in flight at teardown
            for (int64_t j = i - 1; j >= 0 && j >= i - kSmallStages; --j)
                mbar_wait_drain(&bars->xfull[j % kSmallStages], (uint32_t)((j / kSmallStages) & 1),
                                err);
        }
    } else if (warp == 1) {
        // ===================== MMA issuer: polls the E-step queue (tile
        // converted, its score buffer read) and the M-step queue (tile's
        // responsibilities written) and issues whichever is ready
        if (lane == 0) {
            const uint32_t id_e = idesc_f16(128, NE, false, false);
            const uint32_t id_m = idesc_f16(128, NM, true, true);
            const uint64_t dA0 = smem_desc(smem_u32(sm + S::A0), 16, 1024, kSwz128);
            const uint64_t dB = smem_desc(smem_u32(sm + S::B0), 16, 1024, kSwz128);
            const uint64_t dAm0 = smem_desc(smem_u32(sm + S::A0), kBlockBytes, 1024, kSwz128);
            const uint64_t dR0 = smem_desc(smem_u32(sm + S::R0), kBlockBytes, 1024, kSwz128);
            int64_t ie = 0, im = 0;          // next tile for the E-step / the M-step
            bool first_m = true;
            bool wait_flush = false;         // the next M-step waits for a flush
            uint32_t flush_ph = 0;
            long long t_last = clock64();
            while (im < my_tiles) {
                bool progressed = false;
                if (ie < my_tiles && ie < im + NG) {
                    const int g = (int)(ie % NG);
                    const uint32_t ph = (uint32_t)((ie / NG) & 1);
                    if (mbar_try_wait(&bars->afull[g], ph) &&
                        mbar_try_wait(&bars->sfree[g], ph ^ 1)) {
                        tc_fence_after();
                        const uint64_t da = dA0 + (uint32_t)((g * S::ATILE) >> 4);
#pragma unroll
                        for (int ks = 0; ks < KE; ++ks) {
                            const int blk = ks / 4, kk = ks % 4;
                            mma_f16(tmem + g * 64,
                                    da + (uint32_t)((blk * kBlockBytes) >> 4) + 2 * kk,
                                    dB + (uint32_t)((blk * NE * 128) >> 4) + 2 * kk, id_e,
                                    ks ? 1u : 0u);
                        }
                        mma_commit(&bars->sfull[g]);
                        ++ie;
                        progressed = true;
                    }
                }
                if (im < ie) {
                    const int g = (int)(im % NG);
                    const uint32_t ph = (uint32_t)((im / NG) & 1);
                    if (wait_flush && mbar_try_wait(&bars->flushdone, flush_ph)) {
                        tc_fence_after();
                        wait_flush = false;
                        first_m = true;   // the flushed statistics start again from zero
                    }
                    if (!wait_flush && mbar_try_wait(&bars->rfull[g], ph)) {
                        tc_fence_after();
                        const uint64_t dam = dAm0 + (uint32_t)((g * S::ATILE) >> 4);
                        const uint64_t dr = dR0 + (uint32_t)((g * S::RTILE) >> 4);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_f16(t_m, dam + (uint32_t)((kk * 2048) >> 4),
                                    dr + (uint32_t)((kk * 2048) >> 4), id_m,
                                    (first_m && kk == 0) ? 0u : 1u);
                        first_m = false;
                        mma_commit(&bars->mfree[g]);
                        if (((im + 1) % kSmallFlush == 0) || im + 1 == my_tiles) {
                            mma_commit(&bars->flushgo);
                            wait_flush = true;
                            flush_ph = (uint32_t)((im / kSmallFlush) & 1);
                        }
                        ++im;
                        progressed = true;
                    }
                }
                if (progressed) {
                    t_last = clock64();
                } else {
                    if (*abort_flag) break;
                    if (clock64() - t_last > kWaitLimitCycles) {
                        set_error(err, GMM_ERR_TIMEOUT);
                        *abort_flag = 1;
                        break;
                    }
                }
            }
            mma_commit(&bars->done);
            mbar_wait_drain(&bars->done, 0, err);   // no MMA in flight at teardown
        }
    } else {
        // ===================== workers: group g, TMEM lane quadrant q
        const int g = (warp - 2) >> 2;
        const int q = warp & 3;
        const int p = q * 32 + lane;                  // point row of the tile
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        uint8_t *At = sm + S::A0 + g * S::ATILE;
        uint8_t *Rt = sm + S::R0 + g * S::RTILE;
        double ll_acc = 0.0;                          // this thread's points, in order
        for (int64_t i = g; i < my_tiles; i += NG) {
            const int64_t t = blockIdx.x + i * gridDim.x;
            const int64_t n = t * kTileP + p;
            const bool valid = n < N;
            const uint32_t ph = (uint32_t)((i / NG) & 1);
            const int st = (int)(i % kSmallStages);
            // ---- convert the point's raw row into [x | x2_hi | x2_lo | 1 | 0]
            if (!mbar_wait(&bars->xfull[st], (uint32_t)((i / kSmallStages) & 1), err, abort_flag))
                break;
            uint4 raw[D / 8];
            {
                const uint8_t *src = sm + S::X0 + st * S::XRAW + (size_t)p * D * sizeof(XT);
#pragma unroll
                for (int c = 0; c < D / 8; ++c)
                    raw[c] = valid ? *reinterpret_cast<const uint4 *>(src + c * 16)
                                   : make_uint4(0u, 0u, 0u, 0u);
            }
            // the operand tile is free once the group's previous M-step is done
            if (i >= NG && !mbar_wait(&bars->mfree[g], ph ^ 1, err, abort_flag)) break;
            {
                // x 2^-s is exact in fp16 (16-bit data, |x| 2^-s < 181); in
                // fp16 x*x rounded is x^2_hi and fma(x, x, -x^2_hi) is the
                // exact residual x^2_lo (both single roundings of exact
                // values, as the fp32 split gives them)
                const float xsf = __int_as_float((127 - __ldg(P.xs_exp)) << 23);
                const float2 xs2 = make_float2(xsf, xsf);
#pragma unroll
                for (int c = 0; c < D / 8; ++c) {
                    const uint32_t wr[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
                    uint32_t wx[4], wh[4], wl[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float2 f;
                        if constexpr (std::is_same<XT, __nv_bfloat16>::value)
                            f = make_float2(__uint_as_float(wr[e] << 16),
                                            __uint_as_float(wr[e] & 0xFFFF0000u));
                        else
                            f = __half22float2(*reinterpret_cast<const __half2 *>(&wr[e]));
                        f = __fmul2_rn(f, xs2);
                        const __half2 h = __floats2half2_rn(f.x, f.y);
                        const __half2 hh = __hmul2(h, h);
                        const __half2 hl = __hfma2(h, h, __hneg2(hh));
                        wx[e] = h2u(h);
                        wh[e] = h2u(hh);
                        wl[e] = h2u(hl);
                    }
                    // x at chunk c, x2_hi at chunk 4 + c of block 0; x2_lo at
                    // chunk c of block 1
                    *reinterpret_cast<uint4 *>(At + swz128_off(p, c)) =
                        make_uint4(wx[0], wx[1], wx[2], wx[3]);
                    *reinterpret_cast<uint4 *>(At + swz128_off(p, D / 8 + c)) =
                        make_uint4(wh[0], wh[1], wh[2], wh[3]);
                    *reinterpret_cast<uint4 *>(At + kBlockBytes + swz128_off(p, c)) =
                        make_uint4(wl[0], wl[1], wl[2], wl[3]);
                }
                // the raw stage is consumed (its values went into the pieces
                // above): order this thread's reads of it before the next
                // bulk copy into the stage (async proxy), then release it
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->xempty[st]);
                // ones (fp16 1.0) at features 96..111, zeros at 112..127
                const uint32_t one = valid ? 0x3C003C00u : 0u;
                *reinterpret_cast<uint4 *>(At + kBlockBytes + swz128_off(p, 4)) =
                    make_uint4(one, one, one, one);
                *reinterpret_cast<uint4 *>(At + kBlockBytes + swz128_off(p, 5)) =
                    make_uint4(one, one, one, one);
                *reinterpret_cast<uint4 *>(At + kBlockBytes + swz128_off(p, 6)) =
                    make_uint4(0u, 0u, 0u, 0u);
                *reinterpret_cast<uint4 *>(At + kBlockBytes + swz128_off(p, 7)) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->afull[g]);
            // ---- scores -> l_n -> responsibilities
            if (!mbar_wait(&bars->sfull[g], ph, err, abort_flag)) break;
            tc_fence_after();
            float y[KP];
            {
                // y_k = (hi_k + lo_k) a_k + b_k, two components per f32x2 op
                uint32_t r[32];
                uint32_t r2[KP == 16 ? 1 : 32];
                tmem_ld32(tmem + lane_base + g * 64, r);
                if constexpr (KP == 32) tmem_ld32(tmem + lane_base + g * 64 + 32, r2);
                tmem_ld_wait();
#pragma unroll
                for (int k = 0; k < KP; k += 2) {
                    const float2 hi = make_float2(__uint_as_float(r[k]), __uint_as_float(r[k + 1]));
                    float2 lo;
                    if constexpr (KP == 16)
                        lo = make_float2(__uint_as_float(r[KP + k]), __uint_as_float(r[KP + k + 1]));
                    else
                        lo = make_float2(__uint_as_float(r2[k]), __uint_as_float(r2[k + 1]));
                    const float2 t = __ffma2_rn(__fadd2_rn(hi, lo),
                                                *reinterpret_cast<const float2 *>(cA + k),
                                                *reinterpret_cast<const float2 *>(cB + k));
                    y[k] = t.x;
                    y[k + 1] = t.y;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->sfree[g]);
            float m = -INFINITY;
#pragma unroll
            for (int k = 0; k < KP; ++k) m = fmaxf(m, y[k]);
            float l = 0.f;
            if (m != -INFINITY) {
#pragma unroll
                for (int k = 0; k < KP; ++k) l += ex2_approx(y[k] - m);
            }
            if (valid && __ldg(P.dcount) > 0) merge_direct(m, l, __ldg(P.dmf + n));
            const float lse2 = valid ? m + log2f(l) : INFINITY;   // padding rows: r = 0
            if (valid) {
                const float lse = lse2 * 0.69314718055994531f;
                if (!(m > -INFINITY)) set_error(err, GMM_ERR_NONFINITE);
                lse_out[n] = lse;
                if (loglik) loglik[n] = lse;
            }
            {
                // responsibilities -> R row p (MN-major, 64 rows per 128-byte
                // block): [big_hi | big_lo | small_hi | small_lo] x KP, fp16
                // pairs packed in 32-bit words (word w: rows 2w, 2w + 1)
                uint32_t rw[2 * KP];
#pragma unroll
                for (int k = 0; k < KP; k += 2) {
                    const float e0 = y[k] - lse2, e1 = y[k + 1] - lse2;
                    const bool b0 = e0 >= -23.f, b1 = e1 >= -23.f;
                    const float w0 = ex2_approx(e0 + (b0 ? 14.f : 38.f));
                    const float w1 = ex2_approx(e1 + (b1 ? 14.f : 38.f));
                    uint32_t hi, lo;
                    split2(w0, w1, hi, lo);
                    // each half only in its own (big / small) rows
                    const uint32_t mb = (b0 ? 0x0000FFFFu : 0u) | (b1 ? 0xFFFF0000u : 0u);
                    rw[k / 2] = hi & mb;
                    rw[(KP + k) / 2] = lo & mb;
                    rw[(2 * KP + k) / 2] = hi & ~mb;
                    rw[(3 * KP + k) / 2] = lo & ~mb;
                }
#pragma unroll
                for (int c = 0; c < 4 * KP / 8; ++c)
                    *reinterpret_cast<uint4 *>(Rt + (c / 8) * kBlockBytes + swz128_off(p, c % 8)) =
                        make_uint4(rw[4 * c], rw[4 * c + 1], rw[4 * c + 2], rw[4 * c + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->rfull[g]);
            // this thread's points of the total log-likelihood, in tile order
            if (valid) ll_acc += (double)(lse2 * 0.69314718055994531f);
            // ---- statistics flush (this group ran the flush tile)
            if (((i + 1) % kSmallFlush == 0) || i + 1 == my_tiles) {
                if (!mbar_wait(&bars->flushgo, (uint32_t)((i / kSmallFlush) & 1), err, abort_flag))
                    break;
                tc_fence_after();
                // lane p of D_M is operand feature p: x (S1, x 2^s), x2_hi /
                // x2_lo (S2, x 2^2s), ones (S0), zero padding; its 4 KP
                // columns are the R row groups, scaled 2^-14 (big) or 2^-38
                // (small).  Flushes before this one: i / kSmallFlush (the
                // first stores, the later ones add).
                const int nf = (int)(i / kSmallFlush);
                const int xs = __ldg(P.xs_exp);
                const int part = p / D;   // 0 x, 1 x2_hi, 2 x2_lo, 3 ones / padding
                const double fx = part == 0 ? exp2i_d(xs) : part == 3 ? 1.0 : exp2i_d(2 * xs);
                double *row = partial + ((size_t)blockIdx.x * kSmallF + p) * NM;
#pragma unroll 1
                for (int cc = 0; cc < NM / 16; ++cc) {
                    uint32_t r[16];
                    tmem_ld16(t_m + lane_base + cc * 16, r);   // warp-collective
                    tmem_ld_wait();
                    const double f = fx * exp2i_d(cc * 16 < 2 * KP ? -14 : -38);
                    if (p < 3 * D + 16) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const double val = (double)__uint_as_float(r[e]) * f;
                            if (nf > 0) atomicAdd(row + cc * 16 + e, val);
                            else row[cc * 16 + e] = val;
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->flushdone);
            }
        }
        // the warp's 32 per-thread sums in a fixed butterfly order
#pragma unroll
        for (int o = 16; o; o >>= 1) ll_acc += __shfl_xor_sync(0xffffffffu, ll_acc, o);
        if (lane == 0) ll_part[(size_t)blockIdx.x * (4 * NG) + (warp - 2)] = ll_acc;
    }

    // ---- teardown: every role has left its loop (all waits are bounded)
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Fixed-order reduction of the small-K kernel's partial rows into the
// statistics layout S0[K] | S1[K x d] | S2[K x d].  One warp per output
// element: lane L sums the CTAs L, L + 32, ... in order (for each, the four
// row groups of the component, then the second S2 part), and the 32 lane
// sums are combined in a fixed butterfly.  The flush already applied every
// scale.  accumulate: add into `stats` (a later point chunk of the step).
template <int KP>
__global__ void __launch_bounds__(256)
gmm_tc_smallk_reduce_kernel(const double *__restrict__ part, int ncta, int K,
                            double *__restrict__ stats, bool accumulate) {
    constexpr int D = kSmallD;
    constexpr int NM = 4 * KP;
    const int w = 1 + 2 * D;
    const int lane = threadIdx.x & 31;
    const int64_t i = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    if (i >= (int64_t)K * w) return;
    int k, f1, f2;   // component, operand feature(s)
    if (i < K) { k = (int)i; f1 = 3 * D; f2 = -1; }
    else if (i < K + K * D) { k = (int)((i - K) / D); f1 = (int)((i - K) % D); f2 = -1; }
    else { k = (int)((i - K - K * D) / D); f1 = D + (int)((i - K - K * D) % D); f2 = f1 + D; }
    double acc = 0.0;
    for (int b = lane; b < ncta; b += 32) {
        const double *blk = part + (size_t)b * kSmallF * NM;
#pragma unroll
        for (int pc = 0; pc < 4; ++pc) acc += __ldg(blk + (size_t)f1 * NM + pc * KP + k);
        if (f2 >= 0) {
#pragma unroll
            for (int pc = 0; pc < 4; ++pc) acc += __ldg(blk + (size_t)f2 * NM + pc * KP + k);
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) stats[i] = accumulate ? stats[i] + acc : acc;
}
