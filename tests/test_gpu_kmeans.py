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
    # inertia: sum of the squared distances to the assigned centroids.  The
    # kernels accumulate it per cluster as sum |x|^2 - 2 c . sum x + n |c|^2
    # in fp64 (the same quantity), whose rounding is relative to
    # sum |x|^2 + n |c|^2: an exactly-zero inertia comes out at a few 2^-53
    # of that, so the bound has a floor of 1e-13 of it.
    X64 = X.astype(np.float64)
    for b in range(X.shape[0]):
        cb = C[b].astype(np.float64)[out["ids"][b]]
        dd = ((X64[b] - cb) ** 2).sum(-1).sum()
        scale = (X64[b] ** 2).sum() + (cb ** 2).sum()
        assert abs(out["inertia"][b] - dd) <= 1e-5 * dd + 1e-13 * scale, (label, b)
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


@pytest.mark.parametrize("dtype", ["f32", "f16"])
def test_tensor_core_exact_ties_across_chunks(g, dtype):
    """d=64 (tensor-core assignment), K=600 (three 256-centroid chunks):
    integer points exactly midway between a pair of centroids, the pairs
    placed in different chunks, halves of a chunk and orders; the lowest
    index must win (the distances are exact in any precision)."""
    from means_clustering_gmm_b200 import _lib
    d, K = 64, 600
    assert _lib.load().kmeans_workspace_size(1, 16, d, K) > 0
    C = np.zeros((1, K, d), np.float32)
    C[0, :, 1] = 50 + np.arange(K)                    # far from every point
    pairs = [(10, 300), (300, 10), (100, 130), (257, 511), (5, 6), (599, 0)]
    X = np.zeros((1, len(pairs), d), np.float32)
    for p, (a, b) in enumerate(pairs):
        X[0, p, 3] = 20 * (p + 1)
        C[0, a] = X[0, p]
        C[0, b] = X[0, p]
        C[0, a, 0] += 1.0
        C[0, b, 0] -= 1.0
    out = g.kmeans_iteration(g.to_device_x(X.reshape(-1, d), dtype).reshape(X.shape), C)
    assert out["err"] == 0
    np.testing.assert_array_equal(out["ids"][0], [min(a, b) for a, b in pairs])
    np.testing.assert_array_equal(out["ids"], oracle.kmeans_step(X, C)["ids"])


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("shape", [(2, 3001, 64, 300), (1, 1000, 128, 1024), (3, 129, 128, 257)])
def test_tensor_core_chunks_and_ragged_tiles(g, dtype, shape):
    """Several centroid chunks, a ragged last point tile and padded centroid
    rows, against the oracle; the CUDA-core assignment agrees off near-ties."""
    B, N, d, K = shape
    rng = np.random.default_rng(B + N + d + K)
    centres = rng.normal(0, 1, size=(B, K, d))
    lab = rng.integers(0, K, size=(B, N))
    X = round_to((np.take_along_axis(centres, lab[..., None], 1) +
                  0.1 * rng.normal(size=(B, N, d))).astype(np.float32), dtype)
    C = np.stack([X[b, rng.choice(N, size=min(K, N), replace=False)] for b in range(B)])
    if C.shape[1] < K:
        C = np.concatenate([C, rng.normal(0, 1, size=(B, K - C.shape[1], d)).astype(np.float32)], 1)
    Xd = g.to_device_x(X.reshape(B * N, d), dtype).reshape(B, N, d)
    out = g.kmeans_iteration(Xd, C)
    assert out["err"] == 0
    ref = _check(out, X, C, f"tc-{shape}-{dtype}")
    simt = g.kmeans_iteration(Xd, C, flags=2)
    tie = near_tie_mask(ref["d1"], ref["d2"])
    assert not ((simt["ids"] != out["ids"]) & ~tie).any()
