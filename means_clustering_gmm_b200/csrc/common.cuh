// Shared definitions of the libgmm_b200 CUDA sources: status codes, the
// device error word, element loads for the three input dtypes and the
// workspace layout helpers.  No arithmetic of the method lives here.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/gmm_b200.h"

namespace gmmb {

// Device error word: the first int of every workspace.  Kernels record the
// first condition they meet with atomicCAS(0 -> code); the host reads and
// clears it in gmm_last_error().
__device__ __forceinline__ void set_error(int *err, int code) {
    if (err) atomicCAS(err, 0, code);
}

__device__ __forceinline__ float to_float(float v) { return v; }
__device__ __forceinline__ float to_float(__half v) { return __half2float(v); }
__device__ __forceinline__ float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ float load_elem(const T *p);
template <> __device__ __forceinline__ float load_elem<float>(const float *p) { return __ldg(p); }
template <> __device__ __forceinline__ float load_elem<__half>(const __half *p) {
    return __half2float(__ldg(p));
}
template <> __device__ __forceinline__ float load_elem<__nv_bfloat16>(const __nv_bfloat16 *p) {
    return __bfloat162float(__ldg(p));
}

// Per-point selection of the best components (soft assignment): a
// descending list of kTopMax (score, id) pairs, ties to the lower id.
constexpr int kTopMax = 8;
__device__ __forceinline__ void topr_insert(float (&ts)[kTopMax], int (&ti)[kTopMax], float y,
                                            int id) {
#pragma unroll
    for (int j = 0; j < kTopMax; ++j) {
        const bool sw = y > ts[j] || (y == ts[j] && id < ti[j] && y > -INFINITY);
        const float t = ts[j];
        const int u = ti[j];
        ts[j] = sw ? y : t;
        ti[j] = sw ? id : u;
        y = sw ? t : y;
        id = sw ? u : id;
    }
}

constexpr size_t kAlign = 256;
__host__ __device__ inline size_t align_up(size_t v, size_t a = kAlign) {
    return (v + a - 1) / a * a;
}

// Number of blocks the CUDA-core statistics sweep spreads over (a multiple
// of the 148 SMs of a B200); the workspace is sized from it, so it is a
// constant rather than a device query.
constexpr int kSimtTargetBlocks = 4 * 148;

// Fixed tile sizes of the CUDA-core kernels.
constexpr int kLseTileP = 64;     // points per block tile in the LSE sweep
constexpr int kLseTileK = 64;     // components per chunk in the LSE sweep
constexpr int kLseTileJ = 32;     // features per smem chunk
constexpr int kStatsTileP = 32;   // points per tile in the statistics sweep

struct GmmSimtPlan {
    int groups;      // feature groups of 16 per thread row
    int tk;          // components per block
    int kchunks;     // ceil(K / tk)
    int ranges;      // point ranges
    int64_t range_pts;
    int64_t lse_tiles;
};

inline GmmSimtPlan gmm_simt_plan(int64_t N, int d, int K) {
    GmmSimtPlan p;
    p.groups = (d + 15) / 16;
    p.tk = 256 / p.groups;
    if (p.tk > K) p.tk = K;
    p.kchunks = (K + p.tk - 1) / p.tk;
    int r = (kSimtTargetBlocks + p.kchunks - 1) / p.kchunks;
    int64_t max_r = (N + kStatsTileP - 1) / kStatsTileP;
    if (r > max_r) r = (int)max_r;
    if (r < 1) r = 1;
    p.ranges = r;
    int64_t rp = (N + r - 1) / r;
    p.range_pts = (rp + kStatsTileP - 1) / kStatsTileP * kStatsTileP;
    p.lse_tiles = (N + kLseTileP - 1) / kLseTileP;
    return p;
}

// Process-wide tracing state (abi.cu): launch counter and the optional
// kernel timer events recorded around the dominant kernel of a call (the
// caller's pair, or one pair of the library's own per region while the
// collecting timer runs).
void note_launches(int n);
void timer_begin(cudaStream_t s);
void timer_end(cudaStream_t s);
// Suspend (true) or resume the timer in both forms; returns the previous
// state.  gmm_fit suspends it while it captures a graph body, which cannot
// hold event records.
bool timer_suspend(bool suspend);

}  // namespace gmmb
