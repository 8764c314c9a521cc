// Tensor-core (tcgen05 / TMEM) fused GMM E-step.
#include "common.cuh"
#include "kernels.h"

namespace gmmb {

bool gmm_tc_supported(gmm_dtype dt, int64_t N, int d, int K, uint32_t flags) {
    (void)dt; (void)N; (void)d; (void)K; (void)flags;
    return false;
}
int gmm_tc_regime(gmm_dtype dt, int64_t N, int d, int K, uint32_t flags) {
    (void)dt; (void)N; (void)d; (void)K;
    return (flags & GMM_FLAG_FORCE_TWO_SWEEP) ? 2 : 1;
}
size_t gmm_tc_ws_bytes(int64_t N, int d, int K) { (void)N; (void)d; (void)K; return 0; }
int64_t gmm_tc_max_partials(int64_t N, int d, int K) { (void)N; (void)d; (void)K; return 0; }
int64_t gmm_tc_max_ll(int64_t N, int d, int K) { (void)N; (void)d; (void)K; return 0; }

cudaError_t launch_gmm_tc(const void *X, gmm_dtype dt, int64_t N, int d, int K,
                          const float *means, const float *vars, const float *logw,
                          const GmmWs &w, float *loglik, uint32_t flags, int *num_partials,
                          int64_t *num_ll, cudaStream_t s) {
    (void)X; (void)dt; (void)N; (void)d; (void)K; (void)means; (void)vars; (void)logw; (void)w;
    (void)loglik; (void)flags; (void)num_partials; (void)num_ll; (void)s;
    return cudaErrorNotSupported;
}

}  // namespace gmmb
