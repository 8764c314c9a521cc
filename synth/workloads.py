"""Workload definitions and seeded generators (see the package docstring)."""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    number: int
    name: str
    kind: str          # "gmm" or "kmeans"
    N: int             # points (per problem for k-means)
    d: int
    K: int
    dtype: str         # "f32", "bf16", "f16"
    B: int = 1         # independent problems (k-means)
    iters: int = 1
    mean_dist: str = "normal4"   # how component means are drawn
    sigma_lo: float = 0.3
    sigma_hi: float = 1.0
    sigma_fixed: float | None = None
    weights: str = "dirichlet1"  # "equal", "dirichlet1", "dirichlet2"

    @property
    def data_seed(self) -> int:
        return 1000 + self.number

    @property
    def init_seed(self) -> int:
        return 2000 + self.number


# The five workloads: shapes, value distributions and dtypes as specified for
# the fused EM iteration and the Lloyd iteration.
WORKLOADS = {
    1: Workload(1, "gmm-n4096-d16-k8-f32", "gmm", 4096, 16, 8, "f32", iters=1,
                mean_dist="uniform5", sigma_lo=0.5, sigma_hi=1.5, weights="equal"),
    2: Workload(2, "gmm-n1m-d128-k256-f32", "gmm", 1_000_000, 128, 256, "f32", iters=10,
                mean_dist="normal4", sigma_lo=0.3, sigma_hi=1.0, weights="dirichlet1"),
    3: Workload(3, "gmm-n16m-d32-k16-bf16", "gmm", 16_777_216, 32, 16, "bf16", iters=1,
                mean_dist="uniform8", sigma_fixed=1.0, weights="dirichlet2"),
    4: Workload(4, "kmeans-b32-n65536-d128-k1024-f16", "kmeans", 65_536, 128, 1024, "f16",
                B=32, iters=1),
    5: Workload(5, "gmm-n10m-d128-k4096-bf16", "gmm", 10_000_000, 128, 4096, "bf16", iters=1,
                mean_dist="normal4", sigma_lo=0.3, sigma_hi=1.0, weights="dirichlet1"),
}


def round_to(x32: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values once to the stored dtype; returns the rounded values
    as float32 (exactly representable) so both sides can widen them exactly."""
    if dtype == "f32":
        return np.ascontiguousarray(x32, dtype=np.float32)
    import torch
    tdt = {"bf16": torch.bfloat16, "f16": torch.float16}[dtype]
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32))
    return t.to(tdt).to(torch.float32).numpy()


def _component_params(w: Workload, rng: np.random.Generator, K: int, d: int):
    if w.mean_dist == "uniform5":
        mu = rng.uniform(-5.0, 5.0, size=(K, d))
    elif w.mean_dist == "uniform8":
        mu = rng.uniform(-8.0, 8.0, size=(K, d))
    elif w.mean_dist == "normal4":
        mu = rng.normal(0.0, 2.0, size=(K, d))       # N(0, 4 I)
    else:
        raise ValueError(w.mean_dist)
    if w.sigma_fixed is not None:
        sigma = np.full((K, d), w.sigma_fixed)
    else:
        sigma = rng.uniform(w.sigma_lo, w.sigma_hi, size=(K, d))
    if w.weights == "equal":
        wts = np.full(K, 1.0 / K)
    elif w.weights == "dirichlet1":
        wts = rng.dirichlet(np.ones(K))
    elif w.weights == "dirichlet2":
        wts = rng.dirichlet(np.full(K, 2.0))
    else:
        raise ValueError(w.weights)
    return mu, sigma, wts


def gmm_data(w: Workload, N: int | None = None, chunk: int = 1 << 20, shard: int = 0):
    """Draw the mixture data for workload ``w`` (optionally only the first N
    points of the same stream).  Returns (X rounded as float32 [N, d],
    labels [N], true means, true sigmas, true weights).  ``shard`` > 0 draws
    another point stream (seed [data_seed, shard]) from the same mixture, for
    the per-GPU shards of a multi-GPU run."""
    rng = np.random.default_rng(w.data_seed)
    K, d = w.K, w.d
    mu, sigma, wts = _component_params(w, rng, K, d)
    if shard:
        rng = np.random.default_rng([w.data_seed, shard])
    N = w.N if N is None else N
    X = np.empty((N, d), dtype=np.float32)
    labels = np.empty(N, dtype=np.int32)
    cdf = np.cumsum(wts)
    cdf[-1] = 1.0
    mu32 = mu.astype(np.float32)
    sg32 = sigma.astype(np.float32)
    for s in range(0, N, chunk):
        e = min(N, s + chunk)
        u = rng.random(e - s)
        lab = np.searchsorted(cdf, u, side="right").astype(np.int32)
        np.minimum(lab, K - 1, out=lab)
        z = rng.standard_normal((e - s, d), dtype=np.float32)
        X[s:e] = mu32[lab] + sg32[lab] * z
        labels[s:e] = lab
    X = round_to(X, w.dtype)
    return X, labels, mu, sigma, wts


def gmm_init(w: Workload, X: np.ndarray, K: int | None = None):
    """K distinct data points as means, unit variances, equal weights.
    Returns float32 (means [K, d], vars [K, d], logw [K])."""
    K = w.K if K is None else K
    rng = np.random.default_rng(w.init_seed)
    idx = rng.choice(X.shape[0], size=K, replace=False)
    means = np.ascontiguousarray(X[np.sort(idx)], dtype=np.float32)
    var = np.ones_like(means, dtype=np.float32)
    logw = np.full(K, -np.log(K), dtype=np.float32)
    return means, var, logw


def kmeans_data(w: Workload, B: int | None = None, N: int | None = None):
    """B problems of N points drawn from K blobs (centres ~ N(0, I), sigma 0.1).
    Returns X rounded as float32 [B, N, d]."""
    B = w.B if B is None else B
    N = w.N if N is None else N
    rng = np.random.default_rng(w.data_seed)
    X = np.empty((B, N, w.d), dtype=np.float32)
    for b in range(B):
        centres = rng.standard_normal((w.K, w.d), dtype=np.float32)
        lab = rng.integers(0, w.K, size=N)
        X[b] = centres[lab] + np.float32(0.1) * rng.standard_normal((N, w.d), dtype=np.float32)
    return round_to(X, w.dtype)


def kmeans_init(w: Workload, X: np.ndarray, K: int | None = None):
    """Per problem, K distinct points of that problem as initial centroids
    (float32 [B, K, d])."""
    K = w.K if K is None else K
    rng = np.random.default_rng(w.init_seed)
    B, N, d = X.shape
    C = np.empty((B, K, d), dtype=np.float32)
    for b in range(B):
        idx = rng.choice(N, size=K, replace=False)
        C[b] = X[b, np.sort(idx)]
    return C
