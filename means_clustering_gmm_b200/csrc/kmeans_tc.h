// Tensor-core (tcgen05) assignment kernel of Lloyd k-means: interface.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace gmmb {

// Assignment tiles per problem used by the tensor-core kernel (sizes the
// inertia partials of the workspace).
int km_tc_tiles_per_problem(int64_t N);
// Bytes of per-problem centroid pieces the tensor-core kernel keeps in the
// workspace.
size_t km_tc_param_bytes(int B, int d, int K);
// Launches the tensor-core assignment if the shape has a kernel; sets
// *done = false (and launches nothing) otherwise.
cudaError_t launch_km_tc_assign(const void *X, int elem_bytes, int B, int64_t N, int d, int K,
                                const float *C, int32_t *ids, float *mind, double *inpart,
                                int tiles_stride, void *param_ws, int *err, int *used_tiles,
                                bool *done, cudaStream_t s);

}  // namespace gmmb
