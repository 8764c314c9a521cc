"""B200-native fused diagonal-GMM EM and Lloyd k-means (sm_100a, C-ABI library).

The computation lives in ``_lib/libgmm_b200.so`` (CUDA kernels behind the C ABI
of ``include/gmm_b200.h``); this package is its thin torch-facing binding.
"""
from .api import (GMM_FLAG_FORCE_SIMT, GMM_FLAG_FORCE_TWO_SWEEP, GMM_FLAG_NONE,
                  BatchedWorkspace, GmmError, KernelTimer, Workspace, gmm_em_step_batched,
                  gmm_finalize_batched, em_iteration, fit, fit_workspace_size, gmm_em_step, gmm_finalize,
                  gmm_last_error, gmm_workspace_size, init_kmeans, init_kmeans_workspace_size,
                  kmeans_step, kmeans_workspace_size, point_chunk, set_point_chunk,
                  soft_assign)

__all__ = ["GMM_FLAG_FORCE_SIMT", "GMM_FLAG_FORCE_TWO_SWEEP", "GMM_FLAG_NONE",
           "BatchedWorkspace", "gmm_em_step_batched", "gmm_finalize_batched", "GmmError",
           "Workspace", "em_iteration", "fit", "fit_workspace_size", "gmm_em_step",
           "gmm_finalize", "gmm_last_error", "gmm_workspace_size", "init_kmeans",
           "init_kmeans_workspace_size", "kmeans_step", "kmeans_workspace_size", "soft_assign",
           "KernelTimer", "point_chunk", "set_point_chunk"]
