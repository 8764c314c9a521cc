// Tensor-core (tcgen05) assignment kernel of Lloyd k-means: interface.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gmm_b200.h"

namespace gmmb {

// Assignment tiles per problem used by the tensor-core kernel (sizes the
// inertia partials of the workspace).
int km_tc_tiles_per_problem(int64_t N);
// Bytes of per-problem centroid pieces the tensor-core kernel keeps in the
// workspace.
size_t km_tc_param_bytes(int B, int d, int K);
// Launches the tensor-core assignment (centroid pieces, then the assignment
// kernel) if the shape has a kernel (d = 64 or 128) and sets *done; otherwise
// launches nothing and sets *done = false.
cudaError_t launch_km_tc_assign(const void *X, gmm_dtype dt, int B, int64_t N, int d, int K,
                                const float *C, int32_t *ids, void *param_ws, int *err,
                                bool *done, cudaStream_t s);

}  // namespace gmmb
