"""Parity of the Lloyd k-means step (CUDA path, through the C ABI) with the
float64 oracle on the same seeded inputs."""
import numpy as np
import pytest

import oracle
from synth import WORKLOADS, kmeans_data, kmeans_init, round_to

from .parity import TOL_CENTROID, near_tie_mask, normwise

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    from . import gpu_helpers
    return gpu_helpers


def _check(out, X, C, label):
    ref = oracle.kmeans_step(X, C)
    tie = near_tie_mask(ref["d1"], ref["d2"])
    mism = (out["ids"] != ref["ids"]) & ~tie
    assert not mism.any(), (label, int(mism.sum()), int(tie.sum()))
    # the update, teacher-forced on the GPU's own ids
    Co, cnt = oracle.kmeans_update(X, out["ids"], C)
    assert normwise(out["centroids"], Co) <= TOL_CENTROID, label
    assert normwise(out["centroids"], Co) <= 1e-6, label   # fp64 sums: much tighter
    np.testing.assert_array_equal(out["counts"], cnt)
    # inertia: sum of the squared distances to the assigned centroids
    X64 = X.astype(np.float64)
    for b in range(X.shape[0]):
        dd = ((X64[b] - C[b].astype(np.float64)[out["ids"][b]]) ** 2).sum(-1).sum()
        assert out["inertia"][b] == pytest.approx(dd, rel=1e-5)
    return ref


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("shape", [(1, 1, 1, 1), (2, 5000, 20, 37), (3, 2049, 128, 64),
                                   (1, 300, 7, 500)])
def test_ragged_shapes(g, dtype, shape):
    B, N, d, K = shape
    rng = np.random.default_rng(B * 11 + N + d + K)
    X = round_to(rng.normal(0, 1, size=(B, N, d)).astype(np.float32), dtype)
    C = np.stack([X[b, rng.choice(N, size=min(K, N), replace=False)] for b in range(B)])
    if C.shape[1] < K:   # more clusters than points: the rest start far away (empty)
        extra = rng.normal(50, 1, size=(B, K - C.shape[1], d)).astype(np.float32)
        C = np.concatenate([C, extra], axis=1)
    out = g.kmeans_iteration(g.to_device_x(X.reshape(B * N, d), dtype).reshape(B, N, d), C)
    assert out["err"] == 0
    _check(out, X, C, f"{shape}-{dtype}")


def test_exact_ties_go_to_lowest_index(g):
    """Integer-valued points midway between centroid pairs: exact ties in
    any precision; the lowest index must win."""
    X = np.array([[[0, 0], [2, 0], [4, 4], [1, 1]]], dtype=np.float32)
    C = np.array([[[1, 0], [-1, 0], [3, 0], [4, 3], [4, 5], [1, 1]]], dtype=np.float32)
    out = g.kmeans_iteration(g.to_device_x(X.reshape(-1, 2), "f16").reshape(1, 4, 2), C)
    ref = oracle.kmeans_step(X, C)
    np.testing.assert_array_equal(out["ids"], ref["ids"])
    np.testing.assert_array_equal(out["ids"][0], [0, 0, 3, 5])


def test_skewed_cluster_sizes(g):
    """Most points in one cluster (a long segment) and many empty clusters."""
    rng = np.random.default_rng(31)
    X = np.concatenate([rng.normal(0, 0.01, size=(60000, 16)),
                        rng.normal(5, 1, size=(5536, 16))]).astype(np.float32)[None]
    C = np.concatenate([X[:, :1], rng.normal(9, 1, size=(1, 255, 16)).astype(np.float32)], 1)
    out = g.kmeans_iteration(g.to_device_x(X.reshape(-1, 16), "f32").reshape(1, -1, 16), C)
    _check(out, X, C, "skewed")


def test_bitwise_deterministic(g):
    w = WORKLOADS[4]
    X = kmeans_data(w, B=2, N=20000)
    C = kmeans_init(w, X, K=256)
    Xd = g.to_device_x(X.reshape(-1, w.d), "f16").reshape(2, 20000, w.d)
    a = g.kmeans_iteration(Xd, C)
    b = g.kmeans_iteration(Xd, C)
    for k in ["ids", "centroids", "counts", "inertia"]:
        np.testing.assert_array_equal(a[k], b[k])


def test_workload4_reduced(g):
    """The k-means workload's distributions at B=4, N=16384, K=1024."""
    w = WORKLOADS[4]
    X = kmeans_data(w, B=4, N=16384)
    C = kmeans_init(w, X)
    out = g.kmeans_iteration(g.to_device_x(X.reshape(-1, w.d), "f16").reshape(4, 16384, w.d), C)
    assert out["err"] == 0
    _check(out, X, C, "w4-reduced")


@pytest.mark.slow
def test_workload4_full_size_sampled(g):
    """B=32 x 65536 x 128, K=1024 fp16: ids on 2048 sampled points per problem
    (the oracle computes them one by one), the update teacher-forced on every
    point with the GPU ids, counts exact."""
    w = WORKLOADS[4]
    X = kmeans_data(w)
    C = kmeans_init(w, X)
    out = g.kmeans_iteration(g.to_device_x(X.reshape(-1, w.d), "f16").reshape(X.shape), C)
    assert out["err"] == 0
    rng = np.random.default_rng(41)
    for b in range(w.B):
        idx = rng.choice(w.N, 2048, replace=False)
        ref = oracle.kmeans_step(X[b:b + 1, idx], C[b:b + 1])
        tie = near_tie_mask(ref["d1"], ref["d2"])
        assert not ((out["ids"][b:b + 1, idx] != ref["ids"]) & ~tie).any()
    Co, cnt = oracle.kmeans_update(X, out["ids"], C)
    assert normwise(out["centroids"], Co) <= TOL_CENTROID
    np.testing.assert_array_equal(out["counts"], cnt)
