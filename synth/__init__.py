"""Seeded synthetic inputs for the GMM-EM and Lloyd k-means workloads.

This module draws data and initial parameters only; it holds none of the
method's arithmetic (no scores, responsibilities or statistics).  Both the
CUDA path's tests/benchmark and the float64 oracle consume the arrays it
returns, so the two sides always see identical inputs.

Recipe (numpy ``default_rng`` = PCG64):
  * data seed = 1000 + workload number, init seed = 2000 + workload number;
  * mixture data: labels ~ Categorical(w), x = mu[label] + sigma[label] * z,
    z ~ N(0, I), drawn in float32, then rounded once to the stored dtype
    (bf16/fp16 round-to-nearest-even via torch);
  * GMM init: K distinct points drawn without replacement (init seed),
    variances 1, weights 1/K (log weights -log K);
  * k-means: per problem, K blob centres ~ N(0, I), uniform blob labels,
    x = centre + 0.1 z; init = K distinct points of that problem.
"""
from .workloads import (WORKLOADS, Workload, gmm_data, gmm_init, kmeans_data,
                        kmeans_init, round_to)

__all__ = ["WORKLOADS", "Workload", "gmm_data", "gmm_init", "kmeans_data", "kmeans_init",
           "round_to"]
