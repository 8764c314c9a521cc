// Tensor-core (tcgen05) k-means assignment.
#include "common.cuh"
#include "kmeans_tc.h"

namespace gmmb {

int km_tc_tiles_per_problem(int64_t N) { return (int)((N + 127) / 128); }
size_t km_tc_param_bytes(int B, int d, int K) { (void)B; (void)d; (void)K; return 0; }

cudaError_t launch_km_tc_assign(const void *X, int elem_bytes, int B, int64_t N, int d, int K,
                                const float *C, int32_t *ids, float *mind, double *inpart,
                                int tiles_stride, void *param_ws, int *err, int *used_tiles,
                                bool *done, cudaStream_t s) {
    (void)X; (void)elem_bytes; (void)B; (void)N; (void)d; (void)K; (void)C; (void)ids;
    (void)mind; (void)inpart; (void)tiles_stride; (void)param_ws; (void)err; (void)s;
    *used_tiles = 0;
    *done = false;
    return cudaSuccess;
}

}  // namespace gmmb
