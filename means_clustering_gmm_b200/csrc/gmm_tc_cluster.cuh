// Single-sweep EM iteration for 128 < K <= 256 on a cluster of two CTAs.
// Included by gmm_tc.cu after the shared definitions (TcParams, the
// parameter image, load8, split2, merge_direct) and the sweep-2
// kernel; not a separate translation unit.
//
// "Turbo-GMM: FlashAttention-Inspired GPU-Accelerated Gaussian Mixture
// Model" (abstract) normalises the responsibilities in the same traversal
// as the scores whenever the component axis fits on chip.  At K = 256 the
// statistics of all components (K x (1+2d) fp32) do not fit in one SM's
// TMEM next to the scores, but they do across two: each CTA of a cluster
// pair owns one 128-component slice, and both CTAs process the same
// 128-point tiles.  Per tile:
//   * E-step, component-major as in sweep 2: S^T [comp x pt] =
//     W [comp x pieces] . X [pt x pieces]^T in TMEM (lane = component);
//   * the log-sum-exp over all K components of a point: each worker warp
//     reduces its 32 components (a butterfly across lanes gives the
//     quadrant's max and sum of 2^(y - max) per point), the four quadrant
//     partials of both CTAs are exchanged through distributed shared memory
//     (stores into the peer's buffer, remote mbarrier arrivals), and every
//     CTA combines the eight partials in the same fixed order, so both hold
//     the same l_n bit for bit;
//   * r'_kn = 2^(y - l_n + sig_k) is written back into the warp's own score
//     columns as fp16 pieces hi + lo, the A operand of the M-step
//     D[comp, col] += R^T . [X | X o X] and of S0 = R^T . ones.  The lo
//     piece is needed: with a few hundred points per component a single
//     fp16 weight (2^-11 relative) moves mu and var by more than 1e-5.  S0
//     goes through the same tensor-core accumulation as S1 and S2: the fp32
//     accumulator truncates, and the resulting relative bias (about 1e-5
//     over a CTA's tiles) cancels in the quotients S1/S0, S2/S0 only if all
//     three carry it.
// Sixteen worker warps: four TMEM lane quadrants x four 32-point groups, so
// every point of the tile is handled at once; the two 64-point halves are
// released to the M-step separately.  The M-step takes the products with
// the lo X pieces first and releases those pieces, so the next tile's lo
// pieces are stored and its E-step is issued while the products with the hi
// pieces still run (MMAs of one thread execute in issue order, so the
// E-step's writes to the score columns follow the M-step's reads of r').
// TMEM columns: scores / r' [0, 128), S0 [128, 144), the slice's W1_hi
// piece [144, 144 + 32 NB) (loaded once: the E-step takes it as the A
// operand from TMEM, so the parameter ring streams the other pieces only),
// statistics [256, 256 + 2d).
namespace {

constexpr int kClu = 2;            // CTAs per cluster = 128-component slices
constexpr int kWorkersC = 16;      // worker warps
constexpr int kThreadsC = (2 + kWorkersC) * 32;

// The parameter stages the ring streams for one tile, in the order the
// E-step takes them (W1_hi is resident in TMEM):
//   phase 1a: W2_hi b (with x2_lo; W1_hi from TMEM with x_lo before it)
//   phase 1b: W1_lo b, W2_lo b (with x_hi, x2_hi)
//   phase 2:  W2_hi b (with x2_hi, interleaved with W1_hi from TMEM with x_hi)
// The order of the products (small ones first) is the sweep kernels'.
template <int NB>
struct RingC {
    static constexpr int kStages = 4 * NB;
    __device__ static void stage(int i, int &pc, int &b) {
        if (i < NB) {
            pc = 2;
            b = i;
        } else if (i < 3 * NB) {
            const int t = i - NB;
            b = t / 2;
            pc = (t % 2 == 0) ? 1 : 3;
        } else {
            pc = 2;
            b = i - 3 * NB;
        }
    }
};
constexpr int kW1Col = 144;   // TMEM column of the resident W1_hi piece

template <int NB>
struct SmemC {
    static constexpr int XP = 4 * NB * kBlockBytes;   // X pieces: B operand of both contractions
    static constexpr int STAGE = kSlice * 128;        // one parameter stage (16 KB)
    static constexpr int RING = XP;
    static constexpr int NSTAGE = (NB == 2) ? 4 : 8;
    // (max, sum) partials of every quadrant of both CTAs, double-buffered by
    // tile parity: [parity 2][half 2][rank kClu][quadrant 4][64 points] float2
    static constexpr int XBUF = RING + NSTAGE * STAGE;
    static constexpr int XBUF_BYTES = 2 * 2 * kClu * 4 * 64 * 8;
    static constexpr int STG = XBUF + XBUF_BYTES;     // per-warp broadcast staging [18][32] float
    static constexpr int PM = STG + (2 + kWorkersC) * 32 * 4;   // group maxima [4][128]
    static constexpr int ONES = PM + 4 * kSlice * 4;  // 16 x 128 B fp16 ones (S0 operand)
    static constexpr int BARS = ONES + 2048;
    static constexpr int MISC = BARS + 512;
    static constexpr int TOTAL = MISC + 256 + 1024;
    static_assert(TOTAL <= 232448, "shared memory budget");
};

struct BarsC {
    uint64_t wfull[8], wempty[8];
    uint64_t xlo_full, xhi_full, xlo_free, xhi_free;
    uint64_t sfull;
    uint64_t rq[2];       // r' of a 64-point half is in TMEM (its 8 warps)
    uint64_t sq[4];       // the 4 point groups of a quadrant: tile maxima posted
    uint64_t xfull[2];    // all partials of a half arrived (both CTAs)
    uint64_t done;
};

// Reduce v[j] (column j of a 32-column block) over the 32 lanes of the warp;
// lane L returns the reduction of column L.  Five exchange stages (31
// shuffles); the combination order depends only on the lane, so the result
// is reproducible.
template <bool kMax>
__device__ __forceinline__ float warp_colreduce32(float (&v)[32], int lane) {
#pragma unroll
    for (int n = 32; n > 1; n >>= 1) {
        const int o = n >> 1;
        const bool up = (lane & o) != 0;
        if (!kMax && o >= 2) {   // sums: two columns per f32x2 add
#pragma unroll
            for (int j = 0; j < o; j += 2) {
                const float s0 = up ? v[j] : v[j + o], s1 = up ? v[j + 1] : v[j + 1 + o];
                const float k0 = up ? v[j + o] : v[j], k1 = up ? v[j + 1 + o] : v[j + 1];
                const float r0 = __shfl_xor_sync(0xffffffffu, s0, o);
                const float r1 = __shfl_xor_sync(0xffffffffu, s1, o);
                const float2 t = __fadd2_rn(make_float2(k0, k1), make_float2(r0, r1));
                v[j] = t.x;
                v[j + 1] = t.y;
            }
        } else {
#pragma unroll
            for (int j = 0; j < o; ++j) {
                const float send = up ? v[j] : v[j + o];
                const float keep = up ? v[j + o] : v[j];
                const float recv = __shfl_xor_sync(0xffffffffu, send, o);
                v[j] = kMax ? fmaxf(keep, recv) : keep + recv;
            }
        }
    }
    return v[0];
}

// Smallest e with x <= 2^e for a normal x > 0 (exact, from the exponent
// bits); -250 for zero or subnormal x (r below 2^-126 never matters).
__device__ __forceinline__ int ceil_log2_pos(float x) {
    const uint32_t b = __float_as_uint(x);
    const int ex = (int)((b >> 23) & 0xFFu);
    if (!(x > 0.f) || ex == 0) return -250;
    return ex - 127 + ((b & 0x7FFFFFu) != 0u ? 1 : 0);
}

// 2^n as a float, exactly, for -126 <= n <= 127.
__device__ __forceinline__ float exp2i(int n) { return __uint_as_float((uint32_t)(n + 127) << 23); }

// hi = fp16(a), lo = fp16(a - hi) for a pair, the subtraction as one f32x2 op.
__device__ __forceinline__ void split2x(float2 a, uint32_t &hi, uint32_t &lo) {
    const __half2 h = __floats2half2_rn(a.x, a.y);
    const float2 hf = __half22float2(h);
    hi = h2u(h);
    const float2 d = __fadd2_rn(a, make_float2(-hf.x, -hf.y));
    lo = h2u(__floats2half2_rn(d.x, d.y));
}

}  // namespace

template <int NB, typename XT, int DX>
__global__ void __launch_bounds__(kThreadsC, 1)
gmm_tc_cluster_kernel(const XT *__restrict__ X, int64_t N, int K, TcParams P,
                      float *__restrict__ lse_out, float *__restrict__ loglik,
                      double *__restrict__ ll_part, double *__restrict__ partial,
                      int64_t tiles_per_range, int *err) {
    using S = SmemC<NB>;
    constexpr int D = NB * 64;
    constexpr bool XEXACT = !std::is_same<XT, float>::value;
    using Ring = RingC<NB>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    BarsC *bars = reinterpret_cast<BarsC *>(sm + S::BARS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S::MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + S::MISC + 4);
    double *llw = reinterpret_cast<double *>(sm + S::MISC + 16);   // [4] warp sums of l_n
    float2 *xbuf = reinterpret_cast<float2 *>(sm + S::XBUF);
    float *stg = reinterpret_cast<float *>(sm + S::STG);
    float *pmx = reinterpret_cast<float *>(sm + S::PM);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const int64_t ntiles = (N + kTileP - 1) / kTileP;
    const int comp0 = (int)rank * kSlice;
    const int64_t t_begin = (int64_t)blockIdx.y * tiles_per_range;
    const int64_t t_end = min(ntiles, t_begin + tiles_per_range);

    if (tid == 0) {
        for (int s = 0; s < S::NSTAGE; ++s) { mbar_init(&bars->wfull[s], 1); mbar_init(&bars->wempty[s], 1); }
        mbar_init(&bars->xlo_full, kWorkersC);
        mbar_init(&bars->xhi_full, kWorkersC);
        mbar_init(&bars->xlo_free, 1);
        mbar_init(&bars->xhi_free, 1);
        mbar_init(&bars->sfull, 1);
        for (int r = 0; r < 2; ++r) {
            mbar_init(&bars->rq[r], kWorkersC / 2);
            mbar_init(&bars->xfull[r], kWorkersC / 2 * 32 * kClu);   // a half's lanes, every CTA
        }
        for (int q = 0; q < 4; ++q) mbar_init(&bars->sq[q], 4);
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
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_s0 = tmem + 128, t_st = tmem + 256, t_w1 = tmem + kW1Col;
    // the statistics start at zero (every M-step MMA accumulates): the four
    // warps of each TMEM lane quadrant clear its rows before any MMA is issued
    for (int i = tid; i < 512; i += kThreadsC)
        reinterpret_cast<uint32_t *>(sm + S::ONES)[i] = 0x3C003C00u;   // fp16 1.0 pairs
    fence_proxy_async_smem();
    if (warp >= 2) {
        const uint32_t lb = (uint32_t)((warp & 3) * 32) << 16;
        for (int cc = ((warp - 2) >> 2) - 1; cc < 2 * (NB * 64) / 16; cc += 4) {   // S0, statistics
            uint32_t z[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) z[i] = 0u;
            tmem_st16((cc < 0 ? t_s0 : t_st + cc * 16) + lb, z);
        }
        if (((warp - 2) >> 2) == 0) {
            // the slice's W1_hi rows into TMEM as the E-step's A operand: lane =
            // component, column q of block b = features (64 b + 2q, 64 b + 2q + 1)
            // (read from the swizzled image: 16-byte chunk c of row k sits at
            // chunk c ^ (k & 7))
            const int kl = (warp & 3) * 32 + lane;
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                const uint8_t *row = P.img + img_off(0, b, comp0 + kl, NB, P.Kp);
                uint32_t w[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(row + ((c ^ (kl & 7)) << 4)));
                    w[4 * c] = u.x;
                    w[4 * c + 1] = u.y;
                    w[4 * c + 2] = u.z;
                    w[4 * c + 3] = u.w;
                }
                tmem_st32(t_w1 + b * 32 + lb, w);
            }
        }
        tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
    // no CTA of the cluster arrives on a peer's barrier before it is initialised
    cluster_sync_all();
    tc_fence_after();

    if (warp == 0) {
        // ===================== parameter-piece producer (the slice's pieces, every tile)
        if (lane == 0) {
            uint32_t g = 0;
            for (int64_t t = t_begin; t < t_end && !*abort_flag; ++t) {
                for (int i = 0; i < Ring::kStages; ++i, ++g) {
                    int pc, b;
                    Ring::stage(i, pc, b);
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
        // ===================== MMA issuer.  One thread issues every MMA, so the
        // per-MMA work is kept to two descriptor adds: base descriptors are
        // built once, the stage program is unrolled at compile time, and the
        // ring slot advances incrementally.
        if (lane == 0) {
            const uint32_t id_e = idesc_f16(128, kTileP, false, false);   // M = comps, N = points
            const uint32_t id_full = idesc_f16(128, 2 * D, false, true);  // A in TMEM, B MN-major
            const uint32_t id_half = idesc_f16(128, D, false, true);
            const uint64_t dX = smem_desc(smem_u32(sm), 16, 1024, kSwz128);            // E: X pieces
            const uint64_t dR = smem_desc(smem_u32(sm + S::RING), 16, 1024, kSwz128);  // E: ring
            const uint64_t dXm = smem_desc(smem_u32(sm), kBlockBytes, 1024, kSwz128);  // M: [X | X o X]
            const uint32_t id_s0 = idesc_f16(128, 16, false, false);
            const uint64_t b_ones = smem_desc(smem_u32(sm + S::ONES), 16, 1024, kSwz128);
            uint32_t slot = 0, sph = 0;   // ring slot of the next stage and its phase parity
            int it = 0;
            for (int64_t t = t_begin; t < t_end; ++t, ++it) {
                const uint32_t dS = tmem;
                bool ok = true;
                if (!mbar_wait(&bars->xlo_full, it & 1, err, abort_flag)) break;
                tc_fence_after();   // X pieces written by the worker threads
                // phases 1a / 1b: the small products.  (Parameter stages arrive
                // by bulk copy, through the async proxy the MMA reads with; the
                // mbarrier wait is the whole synchronisation.)  Phase 1a:
                // W1_hi (TMEM) x x_lo, then W2_hi x x2_lo, per block.
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    if (!XEXACT) {
                        const uint64_t db = dX + (uint32_t)(((2 * NB + b) * kBlockBytes) >> 4);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_f16_tmem_a(dS, t_w1 + b * 32 + kk * 8, db + 2 * kk, id_e,
                                           (b | kk) ? 1u : 0u);
                    }
                    if (!mbar_wait(&bars->wfull[slot], sph, err, abort_flag)) { ok = false; break; }
                    const uint64_t da = dR + slot * (uint32_t)(S::STAGE >> 4);
                    const uint64_t db = dX + (uint32_t)(((3 * NB + b) * kBlockBytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16(dS, da + 2 * kk, db + 2 * kk, id_e,
                                (XEXACT && b == 0 && kk == 0) ? 0u : 1u);
                    mma_commit(&bars->wempty[slot]);
                    if (++slot == S::NSTAGE) { slot = 0; sph ^= 1; }
                }
                if (!ok) break;
                if (!mbar_wait(&bars->xhi_full, it & 1, err, abort_flag)) break;
                tc_fence_after();
                // phase 1b: W1_lo x x_hi, W2_lo x x2_hi, per block
#pragma unroll
                for (int i = 0; i < 2 * NB; ++i) {
                    const int b = i / 2, pa = i % 2;   // (x_hi with W1_lo, x2_hi with W2_lo)
                    if (!mbar_wait(&bars->wfull[slot], sph, err, abort_flag)) { ok = false; break; }
                    const uint64_t da = dR + slot * (uint32_t)(S::STAGE >> 4);
                    const uint64_t db = dX + (uint32_t)(((pa * NB + b) * kBlockBytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) mma_f16(dS, da + 2 * kk, db + 2 * kk, id_e, 1u);
                    mma_commit(&bars->wempty[slot]);
                    if (++slot == S::NSTAGE) { slot = 0; sph ^= 1; }
                }
                if (!ok) break;
                // phase 2: the large products, x (W1_hi from TMEM) and x^2 (W2_hi)
                // terms interleaved per 16 features
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    if (!mbar_wait(&bars->wfull[slot], sph, err, abort_flag)) { ok = false; break; }
                    const uint64_t da2 = dR + slot * (uint32_t)(S::STAGE >> 4);
                    const uint64_t dbx = dX + (uint32_t)(((0 * NB + b) * kBlockBytes) >> 4);
                    const uint64_t dbx2 = dX + (uint32_t)(((1 * NB + b) * kBlockBytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        mma_f16_tmem_a(dS, t_w1 + b * 32 + kk * 8, dbx + 2 * kk, id_e, 1u);
                        mma_f16(dS, da2 + 2 * kk, dbx2 + 2 * kk, id_e, 1u);
                    }
                    mma_commit(&bars->wempty[slot]);
                    if (++slot == S::NSTAGE) { slot = 0; sph ^= 1; }
                }
                if (!ok) break;
                mma_commit(&bars->sfull);
                // M-step.  First the products with the lo X pieces, one 64-point
                // half at a time as the workers release it, then the lo pieces
                // are handed back for the next tile; then the products with the
                // hi pieces.  (The statistics start at zero; every MMA adds.)
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    if (!mbar_wait(&bars->rq[rr], it & 1, err, abort_flag)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int kk = 4 * rr + q;   // points 16kk .. 16kk+15
                        const uint32_t a_hi = dS + 16 * kk;
                        if (XEXACT) {
                            const uint64_t b_sq_lo =
                                dXm + (uint32_t)((3 * NB * kBlockBytes + kk * 2048) >> 4);
                            mma_f16_tmem_a(t_st + D, a_hi, b_sq_lo, id_half, 1u);
                        } else {
                            const uint64_t b_lo =
                                dXm + (uint32_t)((2 * NB * kBlockBytes + kk * 2048) >> 4);
                            mma_f16_tmem_a(t_st, a_hi, b_lo, id_full, 1u);
                        }
                    }
                }
                if (!ok) break;
                mma_commit(&bars->xlo_free);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t a_hi = dS + 16 * kk, a_lo = a_hi + 8;
                    const uint64_t b_hi = dXm + (uint32_t)((kk * 2048) >> 4);
                    mma_f16_tmem_a(t_s0, a_lo, b_ones, id_s0, 1u);
                    mma_f16_tmem_a(t_s0, a_hi, b_ones, id_s0, 1u);
                    mma_f16_tmem_a(t_st, a_lo, b_hi, id_full, 1u);
                    mma_f16_tmem_a(t_st, a_hi, b_hi, id_full, 1u);
                }
                mma_commit(&bars->xhi_free);
            }
            mma_commit(&bars->done);
            mbar_wait_drain(&bars->done, 0, err);
        }
    } else {
        // ===================== workers (warps 2-17): X conversion, the
        // cross-component log-sum-exp and the responsibility pass
        const int wi = warp - 2;
        const int qd = warp & 3;                  // TMEM lane quadrant = components 32qd..
        const int grp = wi >> 2;                  // 32-point group of the tile
        const int half = grp >> 1, h = grp & 1;   // 64-point half, group within it
        const int c0 = 32 * grp;                  // this warp's points of the tile
        const int kl = qd * 32 + lane;            // component within the slice = TMEM lane
        const int k = comp0 + kl;
        const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
        const float ak = __ldg(P.ak + k), bk = __ldg(P.bk + k);
        const int dcount = __ldg(P.dcount);
        float *my_stg = stg + warp * 32;
        int sig = kSigInit;
        int nflush = 0;   // times this CTA's rows went into its fp64 partial
        const int ct = tid - 64;
        constexpr int CPR = DX / 8;   // 16-byte chunks per row of X
        constexpr int CT = kWorkersC * 32;
        constexpr int GROUPS = (kTileP * CPR + CT - 1) / CT;
        static_assert(DX <= D, "feature padding");
        // features DX..D-1 of the block (d < 64) stay zero in every piece
        if constexpr (DX < D) {
            constexpr int PAD = 8 - CPR;   // zero 16-byte chunks per row
            for (int i = ct; i < kTileP * PAD * 4; i += CT) {
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
                const int gi = ct + kWorkersC * 32 * i;
                const int p = gi / CPR, c = gi % CPR;
                const int64_t n = t * kTileP + p;
                if (n < N && gi < kTileP * CPR) {
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
                const int gi = ct + kWorkersC * 32 * i;
                if (gi >= kTileP * CPR) continue;   // d = 16: fewer chunks than threads
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
                const int gi = ct + kWorkersC * 32 * i;
                if (gi >= kTileP * CPR) continue;   // d = 16: fewer chunks than threads
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
        for (int64_t t = t_begin; t < t_end && live; ++t, ++it) {
            // the next tile's rows (one contiguous run) start moving into L2 now
            if (wi == 0 && lane == 0 && t + 1 < t_end) {
                const int64_t n1 = (t + 1) * kTileP;
                const int64_t rows = min((int64_t)kTileP, N - n1);
                bulk_prefetch_l2(X + n1 * DX, (uint32_t)(rows * DX * sizeof(XT)));
            }
            const int64_t n = t * kTileP + c0 + lane;
            const bool valid = n < N;
            const float2 dm = (valid && dcount > 0) ? __ldg(P.dmf + n) : make_float2(-INFINITY, 0.f);
            if (!mbar_wait(&bars->sfull, it & 1, err, abort_flag)) break;
            tc_fence_after();
            float e[32];
            {
                uint32_t s[32];
                tmem_ld32(tmem + lane_base + c0, s);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float2 y = __ffma2_rn(make_float2(__uint_as_float(s[i]), __uint_as_float(s[i + 1])),
                                                make_float2(ak, ak), make_float2(bk, bk));
                    e[i] = y.x;
                    e[i + 1] = y.y;
                }
            }
            // Quadrant partial of point c0 + L (lane L) over the warp's 32
            // components: the max, then the sum of 2^(y - max), each by a
            // butterfly across the lanes.
            float mq;
            {
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = e[i];
                mq = warp_colreduce32<true>(v, lane);
            }
            my_stg[lane] = (mq == -INFINITY) ? 0.f : mq;
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const float4 m4 = *reinterpret_cast<const float4 *>(my_stg + i);
                const float2 d0 = __fadd2_rn(make_float2(e[i], e[i + 1]), make_float2(-m4.x, -m4.y));
                const float2 d1 = __fadd2_rn(make_float2(e[i + 2], e[i + 3]), make_float2(-m4.z, -m4.w));
                e[i] = ex2_approx(d0.x);
                e[i + 1] = ex2_approx(d0.y);
                e[i + 2] = ex2_approx(d1.x);
                e[i + 3] = ex2_approx(d1.y);
            }
            float lq;
            {
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = e[i];
                lq = warp_colreduce32<false>(v, lane);
            }
            // publish (max, sum) of point c0 + lane to every CTA of the cluster
            float2 *xb = xbuf + (it & 1) * (2 * kClu * 4 * 64);
            {
                const float2 *slot = xb + ((half * kClu + rank) * 4 + qd) * 64 + 32 * h + lane;
#pragma unroll
                for (int c = 0; c < kClu; ++c) st_cluster_f2(mapa_u32(slot, c), mq, lq);
#pragma unroll
                for (int c = 0; c < kClu; ++c) mbar_arrive_cluster(mapa_u32(&bars->xfull[half], c));
            }
            if (!mbar_wait_cluster(&bars->xfull[half], it & 1, err, abort_flag)) break;
            // l_n from the 4 x kClu partials, in the same order in every CTA
            float M = -INFINITY, l = 0.f;
            {
                float2 pr[kClu * 4];
#pragma unroll
                for (int j = 0; j < kClu * 4; ++j) {
                    pr[j] = xb[(half * kClu * 4 + j) * 64 + 32 * h + lane];
                    M = fmaxf(M, pr[j].x);
                }
                if (M != -INFINITY) {
#pragma unroll
                    for (int j = 0; j < kClu * 4; ++j)
                        l += (pr[j].x == -INFINITY) ? 0.f : pr[j].y * ex2_approx(pr[j].x - M);
                }
            }
            if (valid && dcount > 0) merge_direct(M, l, dm);
            const float L = valid ? M + __log2f(l) : INFINITY;
            const float lse = L * 0.69314718055994531f;
            // l_n goes to global memory only after this tile's last barrier
            // arrival: a release arrival waits for the thread's earlier global
            // stores to complete, which would hold up the tensor core.
            if (rank == 0 && qd == 0) {
                double ds = valid ? (double)lse : 0.0;
#pragma unroll
                for (int o = 16; o; o >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, o);
                if (lane == 0) llw[grp] = ds;
            }
            // r = 2^(y - max) * 2^(max - l_n), and its largest value per component
            const float gq = (mq == -INFINITY || !(L < INFINITY)) ? 0.f : ex2_approx(mq - L);
            __syncwarp();
            my_stg[lane] = gq;
            __syncwarp();
            float rmax = 0.f;
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const float4 g4 = *reinterpret_cast<const float4 *>(my_stg + i);
                const float2 r0 = __fmul2_rn(make_float2(e[i], e[i + 1]), make_float2(g4.x, g4.y));
                const float2 r1 = __fmul2_rn(make_float2(e[i + 2], e[i + 3]), make_float2(g4.z, g4.w));
                e[i] = r0.x;
                e[i + 1] = r0.y;
                e[i + 2] = r1.x;
                e[i + 3] = r1.y;
                rmax = fmaxf(fmaxf(rmax, fmaxf(r0.x, r0.y)), fmaxf(r1.x, r1.y));
            }
            pmx[grp * kSlice + kl] = rmax;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->sq[qd]);
            if (!mbar_wait(&bars->sq[qd], it & 1, err, abort_flag)) break;
            const double ll_tile = (rank == 0 && qd == 0 && grp == 0)
                                       ? (llw[0] + llw[1]) + (llw[2] + llw[3]) : 0.0;
            // Dynamic scale: r' = r 2^sig_k.  When a tile's largest r' of
            // component k would pass 2^15 (fp16 tops out just below 2^16),
            // sig_k is lowered so that it lands at 2^12, and what the
            // statistics row already holds is rescaled by the same power of
            // two (exact); the 2^3 headroom keeps rescales rare, and values
            // 2^26 below the top are still normal fp16.  The previous tile's
            // M-step completed before this tile's scores did, so the row is
            // idle; the quadrant's four warps share the rescale.
            const int tm = ceil_log2_pos(fmaxf(fmaxf(pmx[kl], pmx[kSlice + kl]),
                                               fmaxf(pmx[2 * kSlice + kl], pmx[3 * kSlice + kl])));
            const int s_new = (tm > 15 - sig) ? 12 - tm : sig;
            const int delta = s_new - sig;
            if (it > 0 && it % kFlushTiles == 0) {
                // bound the fp32 accumulation chain: move the rows into the
                // fp64 partial (at the scale they were accumulated with)
                const double sc = exp2i_d(-sig);
                double *out = partial + (size_t)blockIdx.y * ((size_t)K * (1 + 2 * (size_t)DX));
#pragma unroll 1
                for (int cc = grp - 1; cc < 2 * D / 16; cc += 4)
                    flush_stats_chunk<D, DX>(t_s0 + lane_base, t_st + lane_base, cc, out, K, k, sc,
                                             nflush > 0, true, __ldg(P.xs_exp));
                ++nflush;
            } else if (it > 0 && __any_sync(0xffffffffu, delta < 0)) {
                const float f = exp2i(max(delta, -126));
#pragma unroll 1
                for (int cc = grp - 1; cc < 2 * D / 16; cc += 4) {   // S0, then the statistics
                    const uint32_t ta = (cc < 0 ? t_s0 : t_st + cc * 16) + lane_base;
                    uint32_t r[16];
                    tmem_ld16(ta, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
                    tmem_st16(ta, r);
                }
            }
            // written in place as [r_hi(16 pts), r_lo(16 pts), r_hi(16),
            // r_lo(16)] (8 columns each): the warp's own score columns
            sig = s_new;
            const float fs = exp2i(min(sig, 127));
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                uint32_t o[16];
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                    const int pi = j * 16 + i;
                    split2x(__fmul2_rn(make_float2(e[pi], e[pi + 1]), make_float2(fs, fs)), o[i / 2],
                            o[8 + i / 2]);
                }
                tmem_st16(tmem + lane_base + c0 + 16 * j, o);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->rq[half]);
            if (rank == 0 && qd == 0) {
                if (valid) {
                    if (!(M > -INFINITY)) set_error(err, GMM_ERR_NONFINITE);
                    lse_out[n] = lse;
                    if (loglik) loglik[n] = lse;
                }
                if (grp == 0 && lane == 0) ll_part[t] = ll_tile;
            }
            if (t + 1 < t_end && !convert_tile(t + 1, it + 1)) break;
        }
        // statistics of the slice: lane = component row, the quadrant's four
        // warps sharing the chunks; added to the fp64 partial if a flush
        // already wrote it
        if (mbar_wait(&bars->done, 0, err, abort_flag)) {
            tc_fence_after();
            double *out = partial + (size_t)blockIdx.y * ((size_t)K * (1 + 2 * (size_t)DX));
            const double sc = exp2i_d(-sig);
#pragma unroll 1
            for (int cc = grp - 1; cc < 2 * D / 16; cc += 4)
                flush_stats_chunk<D, DX>(t_s0 + lane_base, t_st + lane_base, cc, out, K, k, sc,
                                         nflush > 0, false, __ldg(P.xs_exp));
        }
    }

    tc_fence_before();
    __syncthreads();
    // no CTA leaves while its peer may still write into its shared memory
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}
