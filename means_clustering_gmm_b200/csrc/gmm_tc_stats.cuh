// Sweep 2 of the two-sweep regime, component-major ("transposed") form.
// Included by gmm_tc.cu after the shared definitions (TcParams, the
// parameter image, EProg, load8, split2); not a separate translation unit.
//
// With l_n known from sweep 1 ("Turbo-GMM: FlashAttention-Inspired
// GPU-Accelerated Gaussian Mixture Model", abstract: the two-pass design
// recomputes the scores), the responsibilities need no reduction across
// components, so the scores of a 128-component slice are computed as
//     S^T [components x points] = W [comp x 6d pieces] . X [points x 6d pieces]^T
// with TMEM lane = component.  Then, per thread (one component, half of the
// tile's points):
//   * r'_nk = 2^(y_kn - l_n + sig_k) is elementwise;
//   * the dynamic scale sig_k only needs a max over the thread's own points
//     (and its partner's half);
//   * r'_hi / r'_lo are written back into the same TMEM columns (points
//     packed two per column), where they are the A operand of the M-step
//     D[comp, col] += R^T[comp, pt] . [X | X o X][pt, col], and of the
//     S0 contraction R^T . ones (S0 goes through the same tensor-core
//     accumulation as S1 and S2, so their rounding stays coherent in the
//     ratios the M-step takes).
// So the responsibilities never touch shared memory, and the parameter ring
// streams without interruption.  TMEM: scores / responsibilities 128
// columns, S0 16, statistics 2d.
namespace {

template <int NB>
struct SmemT {
    static constexpr int XP = 4 * NB * kBlockBytes;   // X pieces: B operand of both contractions
    static constexpr int STAGE = kSlice * 128;        // one parameter stage (16 KB)
    static constexpr int RING = XP;
    static constexpr int NSTAGE = (NB == 2) ? 5 : 9;
    static constexpr int LSE = RING + NSTAGE * STAGE; // [2][128] l_n (log2 units) per tile
    static constexpr int XCH = LSE + 1024;            // [2][128] int tile maxima
    static constexpr int ONES = XCH + 1024;           // 16 x 128 B of fp16 ones (S0 operand)
    static constexpr int BARS = ONES + 2048;
    static constexpr int MISC = BARS + 256;
    static constexpr int TOTAL = MISC + 256 + 1024;
    static_assert(TOTAL <= 232448, "shared memory budget");
};

struct BarsT {
    uint64_t wfull[9], wempty[9];
    uint64_t xlo_full, xhi_full, xlo_free, xhi_free;
    uint64_t sfull;
    uint64_t rq[2];
    uint64_t pair[4];
    uint64_t done;
};

}  // namespace

template <int NB, typename XT, int DX>
__global__ void __launch_bounds__(kThreads, 1)
gmm_tc_stats_kernel(const XT *__restrict__ X, int64_t N, int K, TcParams P,
                    const float *__restrict__ lse_in, double *__restrict__ partial,
                    int64_t tiles_per_range, int *err) {
    using S = SmemT<NB>;
    constexpr int D = NB * 64;
    constexpr bool XEXACT = !std::is_same<XT, float>::value;
    using Prog = EProg<NB, XEXACT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    BarsT *bars = reinterpret_cast<BarsT *>(sm + S::BARS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S::MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + S::MISC + 4);
    float *lse_s = reinterpret_cast<float *>(sm + S::LSE);
    int *tmax = reinterpret_cast<int *>(sm + S::XCH);                  // [2][128]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t ntiles = (N + kTileP - 1) / kTileP;
    const int comp0 = blockIdx.x * kSlice;
    const int64_t t_begin = (int64_t)blockIdx.y * tiles_per_range;
    const int64_t t_end = min(ntiles, t_begin + tiles_per_range);

    if (tid == 0) {
        for (int s = 0; s < S::NSTAGE; ++s) { mbar_init(&bars->wfull[s], 1); mbar_init(&bars->wempty[s], 1); }
        mbar_init(&bars->xlo_full, 8);
        mbar_init(&bars->xhi_full, 8);
        mbar_init(&bars->xlo_free, 1);
        mbar_init(&bars->xhi_free, 1);
        mbar_init(&bars->sfull, 1);
        mbar_init(&bars->rq[0], 4);
        mbar_init(&bars->rq[1], 4);
        for (int q = 0; q < 4; ++q) mbar_init(&bars->pair[q], 2);
        mbar_init(&bars->done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    for (int i = tid; i < 512; i += kThreads)
        reinterpret_cast<uint32_t *>(sm + S::ONES)[i] = 0x3C003C00u;   // fp16 1.0 pairs
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // TMEM columns: scores / responsibilities at 0, S0 at 128, statistics at 256.
    const uint32_t t_s0 = tmem + 128, t_st = tmem + 256;

    if (warp == 0) {
        // ===================== parameter-piece producer (the slice's pieces, every tile)
        if (lane == 0) {
            uint32_t g = 0;
            for (int64_t t = t_begin; t < t_end && !*abort_flag; ++t) {
                for (int i = 0; i < Prog::kStages; ++i, ++g) {
                    int pc, b, pa;
                    Prog::stage(i, pc, b, pa);
                    const int slot = g % S::NSTAGE;
                    if (!mbar_wait(&bars->wempty[slot], ((g / S::NSTAGE) & 1) ^ 1, err, abort_flag))
                        goto producer_done;
                    mbar_arrive_expect_tx(&bars->wfull[slot], S::STAGE);
                    bulk_g2s(sm + S::RING + slot * S::STAGE,
                             P.img + img_off(pc, b, comp0, NB, P.Kp), S::STAGE, &bars->wfull[slot]);
                }
            }
        producer_done:
            for (uint32_t i = 0; i < (uint32_t)S::NSTAGE && i < g; ++i) {
                const uint32_t gg = g - 1 - i;
                mbar_wait_drain(&bars->wfull[gg % S::NSTAGE], (gg / S::NSTAGE) & 1, err);
            }
        }
    } else if (warp == 1) {
        // ===================== MMA issuer (prebuilt descriptors, unrolled stage
        // program: the issuing thread's per-MMA work is two adds)
        if (lane == 0) {
            const uint32_t id_e = idesc_f16(128, kTileP, false, false);   // M = comps, N = points
            const uint32_t id_full = idesc_f16(128, 2 * D, false, true);  // A in TMEM, B MN-major
            const uint32_t id_half = idesc_f16(128, D, false, true);
            const uint32_t id_s0 = idesc_f16(128, 16, false, false);
            const uint64_t b_ones = smem_desc(smem_u32(sm + S::ONES), 16, 1024, kSwz128);
            const uint64_t dX = smem_desc(smem_u32(sm), 16, 1024, kSwz128);
            const uint64_t dR = smem_desc(smem_u32(sm + S::RING), 16, 1024, kSwz128);
            const uint64_t dXm = smem_desc(smem_u32(sm), kBlockBytes, 1024, kSwz128);
            uint32_t slot = 0, sph = 0;
            int it = 0;
            for (int64_t t = t_begin; t < t_end; ++t, ++it) {
                // single score buffer: this tile's E-step starts after the
                // previous M-step released the X pieces, hence after it read R
                const uint32_t dS = tmem;
                bool ok = true;
                if (!mbar_wait(&bars->xlo_full, it & 1, err, abort_flag)) break;
#pragma unroll
                for (int i = 0; i < Prog::kStages1; ++i) {
                    int pc, b, pa;
                    Prog::stage(i, pc, b, pa);
                    if (i == Prog::kStages1a &&
                        !mbar_wait(&bars->xhi_full, it & 1, err, abort_flag)) { ok = false; break; }
                    if (!mbar_wait(&bars->wfull[slot], sph, err, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t da = dR + slot * (uint32_t)(S::STAGE >> 4);
                    const uint64_t db = dX + (uint32_t)(((pa * NB + b) * kBlockBytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16(dS, da + 2 * kk, db + 2 * kk, id_e, (i | kk) ? 1u : 0u);
                    mma_commit(&bars->wempty[slot]);
                    if (++slot == S::NSTAGE) { slot = 0; sph ^= 1; }
                }
                if (!ok) break;
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
                    const uint64_t dw1 = dR + s1 * (uint32_t)(S::STAGE >> 4);
                    const uint64_t dw2 = dR + s2 * (uint32_t)(S::STAGE >> 4);
                    const uint64_t dbx = dX + (uint32_t)(((0 * NB + b) * kBlockBytes) >> 4);
                    const uint64_t dbx2 = dX + (uint32_t)(((1 * NB + b) * kBlockBytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        mma_f16(dS, dw1 + 2 * kk, dbx + 2 * kk, id_e, 1u);
                        mma_f16(dS, dw2 + 2 * kk, dbx2 + 2 * kk, id_e, 1u);
                    }
                    mma_commit(&bars->wempty[s1]);
                    mma_commit(&bars->wempty[s2]);
                }
                if (!ok) break;
                mma_commit(&bars->sfull);
                // M-step over the two point halves as the readers release them
                const uint32_t acc_first = (it == 0) ? 0u : 1u;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    if (!mbar_wait(&bars->rq[hh], it & 1, err, abort_flag)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 4 * hh; kk < 4 * hh + 4; ++kk) {
                        const uint32_t a_hi = dS + 16 * kk, a_lo = a_hi + 8;
                        const uint64_t b_hi = dXm + (uint32_t)((kk * 2048) >> 4);
                        const uint32_t acc0 = (kk == 0) ? acc_first : 1u;
                        mma_f16_tmem_a(t_st, a_hi, b_hi, id_full, acc0);
                        mma_f16_tmem_a(t_s0, a_hi, b_ones, id_s0, acc0);
                        mma_f16_tmem_a(t_s0, a_lo, b_ones, id_s0, 1u);
                        if (XEXACT) {
                            mma_f16_tmem_a(t_st + D, a_hi,
                                           dXm + (uint32_t)((3 * NB * kBlockBytes + kk * 2048) >> 4),
                                           id_half, 1u);
                        } else {
                            mma_f16_tmem_a(t_st, a_hi,
                                           dXm + (uint32_t)((2 * NB * kBlockBytes + kk * 2048) >> 4),
                                           id_full, 1u);
                        }
                        mma_f16_tmem_a(t_st, a_lo, b_hi, id_full, 1u);
                    }
                }
                if (!ok) break;
                mma_commit(&bars->xlo_free);
                mma_commit(&bars->xhi_free);
            }
            mma_commit(&bars->done);
            mbar_wait_drain(&bars->done, 0, err);
        }
    } else {
        // ===================== workers (warps 2-9): X conversion and the
        // component-major responsibility pass
        const int qd = warp & 3;                  // TMEM lane quadrant = components 32qd..
        const int h = (warp - 2) >> 2;            // point half of the tile
        const int kl = qd * 32 + lane;            // component within the slice = TMEM lane
        const int k = comp0 + kl;
        const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
        const float ak = __ldg(P.ak + k), bk = __ldg(P.bk + k);
        int sig = kSigInit;
        int nflush = 0;   // times this CTA's rows went into its fp64 partial
        const int ct = tid - 64;
        constexpr int CPR = DX / 8;   // 16-byte chunks per row of X
        constexpr int GROUPS = kTileP * CPR / 256;
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
            float lsev = INFINITY;   // padding points: r = 0
            if (ct < kTileP && t * kTileP + ct < N) lsev = lse_in[t * kTileP + ct] * kLog2e;
            // X scale 2^-s (the parameter kernel wrote s before this launch)
            const float xsf = __int_as_float((127 - __ldg(P.xs_exp)) << 23);
#pragma unroll
            for (int i = 0; i < GROUPS; ++i)
#pragma unroll
                for (int e = 0; e < 8; ++e) v[i][e] *= xsf;   // exact: 2^-s
            // lo pieces are computed before the buffer is free; only the
            // stores wait for the previous tile's M-step
            uint32_t wl[GROUPS][4], wsl[GROUPS][4];
#pragma unroll
            for (int i = 0; i < GROUPS; ++i) {
                uint32_t dummy;
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const float x0 = v[i][e], x1 = v[i][e + 1];
                    if (!XEXACT) split2(x0, x1, dummy, wl[i][e / 2]);
                    split2(x0 * x0, x1 * x1, dummy, wsl[i][e / 2]);
                }
            }
            if (it > 0 && !mbar_wait(&bars->xlo_free, (it - 1) & 1, err, abort_flag)) return false;
#pragma unroll
            for (int i = 0; i < GROUPS; ++i) {
                const int gi = ct + 256 * i;
                const int p = gi / CPR, c = gi % CPR;
                const int b = c / 8;
                const uint32_t off = swz128_off(p, c % 8);
                if (!XEXACT)
                    *reinterpret_cast<uint4 *>(sm + (2 * NB + b) * kBlockBytes + off) =
                        make_uint4(wl[i][0], wl[i][1], wl[i][2], wl[i][3]);
                *reinterpret_cast<uint4 *>(sm + (3 * NB + b) * kBlockBytes + off) =
                    make_uint4(wsl[i][0], wsl[i][1], wsl[i][2], wsl[i][3]);
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
            if (ct < kTileP) lse_s[(it & 1) * kTileP + ct] = lsev;
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->xhi_full);
            return true;
        };

        int it = 0;
        bool live = t_begin >= t_end || convert_tile(t_begin, 0);
        for (int64_t t = t_begin; t < t_end && live; ++t, ++it) {
            const uint32_t dS = tmem + lane_base;
            if (!mbar_wait(&bars->sfull, it & 1, err, abort_flag)) break;
            // the converters' l_n writes were released on xhi_full
            if (!mbar_wait(&bars->xhi_full, it & 1, err, abort_flag)) break;
            tc_fence_after();
            const float *L = lse_s + (it & 1) * kTileP + h * 64;
            // Pass A: this thread's max over its 32+32 points of log2 r_kn;
            // with the partner's half, the tile maximum of component k.
            float mx = -INFINITY;
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t r[32];
                tmem_ld32(dS + h * 64 + cc * 32, r);
                float lv[32];
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4 *>(lv + i) =
                        *reinterpret_cast<const float4 *>(L + cc * 32 + i);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    mx = fmaxf(mx, fmaf(__uint_as_float(r[i]), ak, bk) - lv[i]);
            }
            tmax[h * kSlice + kl] = (int)ceilf(fmaxf(mx, -250.f));
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->pair[qd]);
            if (!mbar_wait(&bars->pair[qd], it & 1, err, abort_flag)) break;
            // Dynamic scale (see gmm_tc.cu): r' = r * 2^sig_k with the largest
            // r' in [2^14, 2^15]; a lower sig_k rescales what was accumulated.
            const int tm = max(tmax[kl], tmax[kSlice + kl]);
            const int s_new = min(sig, 15 - tm);
            const int delta = s_new - sig;
            if (it > 0 && it % kFlushTiles == 0) {
                // bound the fp32 accumulation chain: the statistics are idle
                // (the previous M-step completed before these scores did);
                // the two point halves' warps share the move into the fp64
                // partial, at the scale the rows were accumulated with
                const double sc = exp2i_d(-sig);
                double *out = partial + (size_t)blockIdx.y * ((size_t)K * (1 + 2 * (size_t)DX));
#pragma unroll 1
                for (int cc = h - 1; cc < 2 * D / 16; cc += 2)
                    flush_stats_chunk<D, DX>(t_s0 + lane_base, t_st + lane_base, cc, out, K, k, sc,
                                             nflush > 0, true, __ldg(P.xs_exp));
                tmem_st_wait();
                ++nflush;
                sig = s_new;
            } else if (h == 0 && it > 0 && __any_sync(0xffffffffu, delta < 0)) {
                // the previous M-step completed before these scores did
                const float f = exp2f((float)delta);
                {
                    uint32_t r[32];
                    tmem_ld32(t_s0 + lane_base, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
                    tmem_st32(t_s0 + lane_base, r);
                }
                for (int cc = 0; cc < 2 * D / 32; ++cc) {
                    uint32_t r[32];
                    tmem_ld32(t_st + lane_base + cc * 32, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
                    tmem_st32(t_st + lane_base + cc * 32, r);
                }
                tmem_st_wait();
            }
            sig = s_new;
            // Pass B: r' for 32 points at a time, written in place as
            // [r_hi(16 pts), r_lo(16 pts), r_hi(16), r_lo(16)] (8 columns each)
            const float fsig = (float)sig;
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t r[32];
                const uint32_t col = h * 64 + cc * 32;
                tmem_ld32(dS + col, r);
                float lv[32];
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4 *>(lv + i) =
                        *reinterpret_cast<const float4 *>(L + cc * 32 + i);
                tmem_ld_wait();
                uint32_t o[32];
#pragma unroll
                for (int j = 0; j < 2; ++j) {        // 16-point group
#pragma unroll
                    for (int i = 0; i < 16; i += 2) {
                        const int pi = j * 16 + i;
                        // the same y as pass A, so y + sig <= 15 (clamped anyway)
                        const float y0 = fmaf(__uint_as_float(r[pi]), ak, bk) - lv[pi];
                        const float y1 = fmaf(__uint_as_float(r[pi + 1]), ak, bk) - lv[pi + 1];
                        uint32_t hi, lo;
                        split2(ex2_approx(fminf(y0 + fsig, 15.f)), ex2_approx(fminf(y1 + fsig, 15.f)),
                               hi, lo);
                        o[j * 16 + i / 2] = hi;
                        o[j * 16 + 8 + i / 2] = lo;
                    }
                }
                tmem_st32(dS + col, o);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->rq[h]);
            if (t + 1 < t_end && !convert_tile(t + 1, it + 1)) break;
        }
        // statistics of the slice: lane = component row, the two halves'
        // warps sharing the chunks; added to the fp64 partial if a flush
        // already wrote it
        if (mbar_wait(&bars->done, 0, err, abort_flag)) {
            tc_fence_after();
            double *out = partial + (size_t)blockIdx.y * ((size_t)K * (1 + 2 * (size_t)DX));
            const double sc = (t_begin < t_end) ? exp2i_d(-sig) : 0.0;   // no tiles: zeros
#pragma unroll 1
            for (int cc = h - 1; cc < 2 * D / 16; cc += 2)
                flush_stats_chunk<D, DX>(t_s0 + lane_base, t_st + lane_base, cc, out, K, k, sc,
                                         nflush > 0, false, __ldg(P.xs_exp));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}
