// Direct-form scoring of the components the expanded (tensor-core) form
// cannot score accurately: their scores and per-point (max, sum), and their
// fp64 statistics.  Included by gmm_tc.cu after the shared definitions
// (load8, merge_direct, kLog2e); not a separate translation unit.
//
// The pages score in the expanded form X . (mu/var)^T plus constants
// ("Flash-GMM: a memory-efficient kernel for scalable soft clustering",
// abstract); for a point near component k its terms are each about
// Q_k = sum_j mu_kj^2 / var_kj while their sum is O(d), so a component with a
// large Q_k is scored here in the same log-density's direct form
// s = c_k + sum_j nhl_kj (x_j - mu_kj)^2, on CUDA cores in fp32.

// a1'': direct-form scores of the listed components, the CUDA-core form
// s_nk = c_k + sum_j nhl_kj (x_nj - mu_kj)^2 (nhl = -1/(2 var),
// c_k = log w_k - 1/2 sum_j log(2 pi var_kj)), in log2 units: dscore[slot][n]
// = s * log2(e), and per point dmf[n] = (max_k, sum_k 2^(y - max)) over the
// listed components.  The list is taken 16 components per pass over X (one
// pass unless more than 16 are listed); a point's (max, sum) is folded over
// the passes in list order.
//
// Two blocks per SM (128 registers a thread: the feature loop keeps more
// loads in flight than at 80).  Every warp works alone on 32-point tiles
// (no block barrier in the tile loop).  It stages 16 features of its 32
// points at a time in its own shared-memory buffer, double-buffered, with
// coalesced loads (whole 64-byte row segments, 16 bytes a lane).  The stage
// is [feature][point] with the point index XOR-ed by a multiple of 4 that
// depends on the feature's 16-byte piece, so the transposing stores and the
// 4-point reads are both free of bank conflicts.  Lane (g, q) owns points 4q..4q+3 of the tile and
// components 4g..4g+3 of the pass: per feature one 16-byte x load and two
// 16-byte (mu, nhl) loads feed 24 fp32x2 operations (x - mu exact-rounded,
// then square and scale: three operations per term, the least that keeps
// x - mu exact).  The four groups' (max, sum) are merged with shuffles.
// The same pass takes max |x| over X for the X scale of the tensor-core
// kernels (into *xmax, zero before the launch); with no listed component the
// kernel does only that.
constexpr int kDirThreads = 256;
constexpr int kDirWarps = kDirThreads / 32;
constexpr int kDirPts = 32;                                 // points per warp tile
constexpr int kDirSlots = 16;                               // components per pass
constexpr int kDirMu = 128 * kDirSlots * 4;                 // [feature][slot] floats
constexpr int kDirStage = 16 * kDirPts * 4;                 // one staged [16][32] block
constexpr int kDirSmem = 2 * kDirMu + kDirWarps * 2 * kDirStage + kDirSlots * 4;

// 16 bytes of a row: 4 fp32 or 8 16-bit features, as floats
template <typename XT>
__device__ __forceinline__ void load_piece(const XT *p, float *v) {
    if constexpr (sizeof(XT) == 4) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    } else {
        float t[8];
        load8<XT>(p, t);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = t[i];
    }
}

template <typename XT>
__global__ void __launch_bounds__(kDirThreads, 2)
gmm_tc_direct_scores_kernel(const XT *__restrict__ X, int64_t N, int d,
                            const float *__restrict__ means, const float *__restrict__ vars,
                            const float *__restrict__ logw, const int *__restrict__ dlist,
                            const int *__restrict__ dcount, float *__restrict__ dscore,
                            float2 *__restrict__ dmf, uint32_t *__restrict__ xmax) {
    constexpr int PF = 16 / (int)sizeof(XT);   // features per 16-byte piece
    constexpr int PPR = 16 / PF;               // pieces per point and 16-feature block
    constexpr int PPL = kDirPts * PPR / 32;    // pieces per lane and block
    constexpr int XS = kDirPts / PPR;          // swizzle unit: 8 (fp32) or 16 (16-bit)
    extern __shared__ __align__(16) uint8_t dsm[];
    float *Mu = reinterpret_cast<float *>(dsm);                     // -mu   [128][kDirSlots]
    float *Nh = Mu + 128 * kDirSlots;                               // nhl   [128][kDirSlots]
    float *St = Nh + 128 * kDirSlots;                               // [warp][2][16][32]
    float *cs = St + kDirWarps * 2 * (kDirStage / 4);               // [kDirSlots]
    const int cnt = *dcount;
    if (cnt == 0) {   // nothing to score: max |x| alone
        block_max_to(xmax_scan<XT>(X, N * (int64_t)d, blockIdx.x * (int64_t)blockDim.x + threadIdx.x,
                                   (int64_t)gridDim.x * blockDim.x),
                     xmax);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t xm = 0;   // max |x| of what this thread fetched in the first pass
    const int q = lane & 7, grp = lane >> 3;   // points 4q..4q+3, components 4grp..4grp+3
    float *st = St + warp * 2 * (kDirStage / 4);
    const int nblk = d / 16;
    const int64_t ntiles = (N + kDirPts - 1) / kDirPts;
    const int64_t gwarp = (int64_t)blockIdx.x * kDirWarps + warp;
    const int64_t nwarps = (int64_t)gridDim.x * kDirWarps;
    float v[PPL * PF];   // staging: pieces lane + 32 i; piece u = point u / PPR, part u % PPR
    bool first = true;   // the first pass sees every element of X once
    auto fetch = [&](int64_t tile, int j0) {
#pragma unroll
        for (int i = 0; i < PPL; ++i) {
            const int u = lane + 32 * i;
            const int64_t nn = tile * kDirPts + u / PPR;
            if (tile < ntiles && nn < N) {
                load_piece<XT>(X + nn * d + j0 + (u % PPR) * PF, v + i * PF);
            } else {
#pragma unroll
                for (int e = 0; e < PF; ++e) v[i * PF + e] = 0.f;
            }
        }
        if (first) {
#pragma unroll
            for (int e = 0; e < PPL * PF; ++e) xm = max(xm, abs_bits(v[e]));
        }
    };
    uint32_t g = 0;   // staged-block counter (buffer parity)
    for (int b0 = 0; b0 < cnt; b0 += kDirSlots) {
        const int pc = min(kDirSlots, cnt - b0);   // components in this pass
        __syncthreads();                           // the previous pass is done with Mu, Nh, cs
        for (int i = tid; i < d * kDirSlots; i += kDirThreads) {
            const int j = i / kDirSlots, b = i % kDirSlots;
            float mu = 0.f, nh = 0.f;   // padding slots: score 0, never stored
            if (b < pc) {
                const size_t off = (size_t)dlist[b0 + b] * d + j;
                mu = means[off];
                nh = -0.5f / vars[off];
            }
            Mu[i] = -mu;
            Nh[i] = nh;
        }
        for (int b = warp; b < pc; b += kDirWarps) {
            const int k = dlist[b0 + b];
            double acc = 0.0;
            for (int j = lane; j < d; j += 32) acc += log(2.0 * M_PI * (double)vars[(size_t)k * d + j]);
#pragma unroll
            for (int w = 16; w; w >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w);
            if (lane == 0) cs[b] = (float)((double)logw[k] - 0.5 * acc);
        }
        __syncthreads();
        int64_t tile = gwarp;
        fetch(tile, 0);
        for (; tile < ntiles; tile += nwarps) {
            // [component of the group][points (4q, 4q+1) | (4q+2, 4q+3)]
            float2 acc[4][2];
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[c][0] = acc[c][1] = make_float2(0.f, 0.f);
            for (int blk = 0; blk < nblk; ++blk, ++g) {
                float *xb = st + (g & 1) * (kDirStage / 4);
#pragma unroll
                for (int i = 0; i < PPL; ++i) {
                    const int u = lane + 32 * i;
                    const int p = u / PPR, c = u % PPR;
#pragma unroll
                    for (int e = 0; e < PF; ++e)
                        xb[(c * PF + e) * kDirPts + (p ^ (XS * c))] = v[i * PF + e];
                }
                __syncwarp();
                if (blk + 1 < nblk) fetch(tile, (blk + 1) * 16);
                else fetch(tile + nwarps, 0);
                const float *mr = Mu + blk * 16 * kDirSlots + 4 * grp;
                const float *nr = Nh + blk * 16 * kDirSlots + 4 * grp;
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    const float4 xv = *reinterpret_cast<const float4 *>(
                        xb + jj * kDirPts + ((4 * q) ^ (XS * (jj / PF))));
                    const float4 m = *reinterpret_cast<const float4 *>(mr + jj * kDirSlots);
                    const float4 hl = *reinterpret_cast<const float4 *>(nr + jj * kDirSlots);
                    const float mm[4] = {m.x, m.y, m.z, m.w}, hh[4] = {hl.x, hl.y, hl.z, hl.w};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float2 mc = make_float2(mm[c], mm[c]), hc = make_float2(hh[c], hh[c]);
                        const float2 d0 = __fadd2_rn(make_float2(xv.x, xv.y), mc);
                        const float2 d1 = __fadd2_rn(make_float2(xv.z, xv.w), mc);
                        acc[c][0] = __ffma2_rn(__fmul2_rn(d0, d0), hc, acc[c][0]);
                        acc[c][1] = __ffma2_rn(__fmul2_rn(d1, d1), hc, acc[c][1]);
                    }
                }
                __syncwarp();   // every lane is done with this buffer before it is refilled
            }
            // scores, and (max, sum) over the lane's components per point
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY}, l[4] = {0.f, 0.f, 0.f, 0.f};
            float y[4][4];   // [component][point]
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int b = 4 * grp + c;
                const float s4[4] = {acc[c][0].x, acc[c][0].y, acc[c][1].x, acc[c][1].y};
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    y[c][p] = b < pc ? (s4[p] + cs[b]) * kLog2e : -INFINITY;
                    mx[p] = fmaxf(mx[p], y[c][p]);
                }
                if (b < pc) {
                    const int64_t n = tile * kDirPts + 4 * q;
                    float *dst = dscore + (size_t)(b0 + b) * N + n;
#pragma unroll
                    for (int p = 0; p < 4; ++p)
                        if (n + p < N) dst[p] = y[c][p];
                }
            }
#pragma unroll
            for (int p = 0; p < 4; ++p) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (y[c][p] != -INFINITY) l[p] += exp2f(y[c][p] - mx[p]);
            }
            // merge the four groups (lanes q, q+8, q+16, q+24) in a fixed pattern
#pragma unroll
            for (int o = 8; o <= 16; o <<= 1) {
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const float mo = __shfl_xor_sync(0xffffffffu, mx[p], o);
                    const float lo = __shfl_xor_sync(0xffffffffu, l[p], o);
                    const float mm = fmaxf(mx[p], mo);
                    if (mm != -INFINITY) {
                        l[p] = (mx[p] == -INFINITY ? 0.f : l[p] * exp2f(mx[p] - mm)) +
                               (mo == -INFINITY ? 0.f : lo * exp2f(mo - mm));
                        mx[p] = mm;
                    }
                }
            }
            if (grp == 0) {
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const int64_t n = tile * kDirPts + 4 * q + p;
                    if (n < N) {
                        float m = -INFINITY, ll = 0.f;
                        if (b0 > 0) {   // what the earlier passes folded (this lane wrote it)
                            const float2 f = dmf[n];
                            m = f.x;
                            ll = f.y;
                        }
                        merge_direct(m, ll, make_float2(mx[p], l[p]));
                        dmf[n] = make_float2(m, ll);
                    }
                }
            }
        }
        first = false;
    }
    block_max_to(xm, xmax);
}

// a4: sufficient statistics of the listed components:
// r_nk = 2^(dscore - l_n log2 e) in fp64 (r >= 2^-126), S0 = sum r,
// S1 = sum r x, S2 = sum r x^2.  Block (b, rr) sums listed component b over point range rr:
// warp w scans the points w*32 + 256 i of the range; for each point with
// r > 0 (ballot) its lanes add the point's features (d/32 each, fp64); the
// warps' sums are combined in warp order into dpart[b][rr], and
// gmm_tc_direct_stats_final adds the ranges in order into the reduced
// statistics.  Reproducible run to run.
constexpr int kDirRanges = 64;
// Responsibilities below 2^-126 are left out of the sums (the tensor-core
// statistics cannot carry them either): a point far from the component then
// costs one score read instead of a row of fp64 products.
constexpr double kDirRMin = -126.0;

template <typename XT>
__global__ void __launch_bounds__(256)
gmm_tc_direct_stats_kernel(const XT *__restrict__ X, int64_t N, int d, int64_t span,
                           const int *__restrict__ dcount, const float *__restrict__ dscore,
                           const float *__restrict__ lse, double *__restrict__ dpart) {
    __shared__ double red[8][1 + 2 * 128];
    const int b = blockIdx.x, rr = blockIdx.y;
    if (b >= *dcount) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int per = d / 32;   // features per lane (2 or 4)
    const int64_t n0 = (int64_t)rr * span, n1 = min(N, n0 + span);
    double s0 = 0.0, s1[4] = {0.0, 0.0, 0.0, 0.0}, s2[4] = {0.0, 0.0, 0.0, 0.0};
    for (int64_t c4 = n0 + warp * 32; c4 < n1; c4 += 256 * 4) {
        // four rounds' scores and l_n in flight at once (the scan is latency-bound)
        float ds[4], ls[4];
#pragma unroll
        for (int rd = 0; rd < 4; ++rd) {
            const int64_t n = c4 + 256 * rd + lane;
            ds[rd] = n < n1 ? dscore[(size_t)b * N + n] : 0.f;
            ls[rd] = n < n1 ? lse[n] : 0.f;
        }
#pragma unroll 1
        for (int rd = 0; rd < 4; ++rd) {
            const int64_t c0 = c4 + 256 * rd;
            const int64_t n = c0 + lane;
            double r = 0.0;
            if (n < n1) {
                const double e = (double)ds[rd] - (double)(ls[rd] * kLog2e);
                r = e > kDirRMin ? exp2(e) : 0.0;
            }
            uint32_t bal = __ballot_sync(0xffffffffu, r > 0.0);
            while (bal) {
                const int src = __ffs(bal) - 1;
                bal &= bal - 1;
                const double ri = __shfl_sync(0xffffffffu, r, src);
                const XT *xr = X + (c0 + src) * d;
                s0 += ri;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (u < per) {
                        const double x = (double)load_elem<XT>(xr + u * 32 + lane);
                        s1[u] += ri * x;
                        s2[u] += ri * x * x;
                    }
                }
            }
        }
    }
    if (lane == 0) red[warp][0] = s0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        if (u < per) {
            red[warp][1 + u * 32 + lane] = s1[u];
            red[warp][1 + d + u * 32 + lane] = s2[u];
        }
    }
    __syncthreads();
    double *out = dpart + ((size_t)b * gridDim.y + rr) * (1 + 2 * (size_t)d);
    for (int i = tid; i < 1 + 2 * d; i += 256) {
        double acc = 0.0;
#pragma unroll
        for (int w = 0; w < 8; ++w) acc += red[w][i];
        out[i] = acc;
    }
}

__global__ void __launch_bounds__(256)
gmm_tc_direct_stats_final(int d, int K, int nranges, const int *__restrict__ dlist,
                          const int *__restrict__ dcount, const double *__restrict__ dpart,
                          double *__restrict__ stats) {
    const int b = blockIdx.x;
    if (b >= *dcount) return;
    const int k = dlist[b];
    const int w = 1 + 2 * d;
    for (int i = threadIdx.x; i < w; i += blockDim.x) {
        double acc = 0.0;
        for (int rr = 0; rr < nranges; ++rr) acc += dpart[((size_t)b * nranges + rr) * w + i];
        if (i == 0) stats[k] += acc;
        else if (i <= d) stats[K + (size_t)k * d + (i - 1)] += acc;
        else stats[K + (size_t)K * d + (size_t)k * d + (i - 1 - d)] += acc;
    }
}

