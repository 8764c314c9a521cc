"""Parity of the fused GMM EM step (CUDA path, through the C ABI) with the
float64 oracle on the same seeded inputs."""
import numpy as np
import pytest

import oracle
from synth import WORKLOADS, gmm_data, gmm_init, round_to

from .parity import (TOL_LOGLIK, TOL_PARAM, check_gmm_iteration, check_stats, loglik_err,
                     normwise)

pytestmark = pytest.mark.gpu

# sum_k S0_k = N holds exactly in real arithmetic (rows of R sum to 1).  The
# tensor core accumulates the statistics in fp32 with truncation, about 6e-9
# relative drift per accumulating MMA; the kernels move them into fp64 every
# 32 tiles, so the drift stays below about 4e-6.  (The per-weight tolerance,
# absolute 1e-5, allows K times more.)
TOL_S0_SUM = 1e-5


@pytest.fixture(scope="module")
def g():
    from . import gpu_helpers
    return gpu_helpers


def _ref(X32, mu, var, lw):
    return oracle.gmm_em_iteration(X32, mu, var, lw)


def _case(rng, N, d, K, dtype, spread=3.0):
    mu_t = rng.normal(0, spread, size=(K, d))
    lab = rng.integers(0, K, size=N)
    X = (mu_t[lab] + rng.uniform(0.4, 1.2, size=(K, d))[lab] *
         rng.standard_normal((N, d))).astype(np.float32)
    X = round_to(X, dtype)
    idx = rng.choice(N, size=K, replace=False)
    mu = X[idx].astype(np.float32)
    var = rng.uniform(0.5, 2.0, size=(K, d)).astype(np.float32)
    w = rng.dirichlet(np.ones(K))
    return X, mu, var, np.log(w).astype(np.float32)


@pytest.mark.parametrize("flags", [0, 2])
def test_workload1_one_iteration(g, flags):
    """4096 x 16, K=8, fp32 (the small workload), one EM iteration."""
    w = WORKLOADS[1]
    X, *_ = gmm_data(w)
    mu, var, lw = gmm_init(w, X)
    out = g.gmm_iteration(g.to_device_x(X, "f32"), mu, var, lw, flags=flags)
    assert out["err"] == 0
    ref = _ref(X, mu, var, lw)
    check_gmm_iteration(out, ref, "f32", "w1")
    assert out["loglik_total"] == pytest.approx(ref["loglik_total"], rel=1e-6)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("shape", [(1, 1, 1), (7, 3, 2), (1000, 37, 5), (3001, 64, 70),
                                   (5000, 128, 33), (2048, 16, 300)])
def test_ragged_shapes(g, dtype, shape):
    """Sizes that are not multiples of any tile, in all three input dtypes."""
    N, d, K = shape
    rng = np.random.default_rng(N * 7 + d * 3 + K)
    X, mu, var, lw = _case(rng, N, d, K, dtype)
    out = g.gmm_iteration(g.to_device_x(X, dtype), mu, var, lw)
    assert out["err"] == 0
    ref = _ref(X, mu, var, lw)
    check_gmm_iteration(out, ref, dtype, f"{shape}-{dtype}")


def test_simt_and_default_paths_agree(g):
    rng = np.random.default_rng(21)
    X, mu, var, lw = _case(rng, 20000, 128, 64, "f32")
    Xd = g.to_device_x(X, "f32")
    a = g.gmm_iteration(Xd, mu, var, lw, flags=0)
    b = g.gmm_iteration(Xd, mu, var, lw, flags=2)
    assert normwise(a["means"], b["means"]) < 1e-5
    assert normwise(a["vars"], b["vars"]) < 1e-5
    assert loglik_err(a["loglik"], b["loglik"]) < 1e-4


def test_bitwise_deterministic(g):
    rng = np.random.default_rng(22)
    X, mu, var, lw = _case(rng, 50000, 64, 40, "f32")
    Xd = g.to_device_x(X, "f32")
    a = g.gmm_iteration(Xd, mu, var, lw)
    b = g.gmm_iteration(Xd, mu, var, lw)
    for k in ["means", "vars", "logw", "loglik", "S0", "S1", "S2"]:
        np.testing.assert_array_equal(a[k], b[k])
    assert a["loglik_total"] == b["loglik_total"]


def test_bitwise_deterministic_cluster(g):
    """The two-CTA single sweep (K = 256): the per-point log-sum-exp is
    combined from both CTAs' partials in a fixed order, so reruns agree bit
    for bit."""
    rng = np.random.default_rng(25)
    X, mu, var, lw = _case(rng, 30000, 128, 256, "f32")
    Xd = g.to_device_x(X, "f32")
    a = g.gmm_iteration(Xd, mu, var, lw)
    b = g.gmm_iteration(Xd, mu, var, lw)
    assert a["err"] == 0
    for k in ["means", "vars", "logw", "loglik", "S0", "S1", "S2"]:
        np.testing.assert_array_equal(a[k], b[k])
    assert a["loglik_total"] == b["loglik_total"]


def test_zero_weight_component_keeps_parameters(g):
    rng = np.random.default_rng(23)
    X, mu, var, lw = _case(rng, 4000, 8, 4, "f32")
    lw = lw.copy()
    lw[2] = -np.inf
    out = g.gmm_iteration(g.to_device_x(X, "f32"), mu, var, lw)
    assert out["err"] == 0
    np.testing.assert_array_equal(out["means"][2], mu[2])
    np.testing.assert_array_equal(out["vars"][2], var[2])
    assert out["logw"][2] == -np.inf
    ref = _ref(X, mu, var, lw)
    check_gmm_iteration(out, ref, "f32", "zero-weight")


def test_identical_points_hit_variance_floor(g):
    X = np.ones((300, 4), dtype=np.float32)
    mu = np.zeros((1, 4), np.float32)
    var = np.ones((1, 4), np.float32)
    out = g.gmm_iteration(g.to_device_x(X, "f32"), mu, var, np.zeros(1, np.float32))
    np.testing.assert_allclose(out["means"], 1.0, rtol=1e-7)
    np.testing.assert_array_equal(out["vars"], np.float32(1e-6))


def test_stats_column_sums_property(g):
    """sum_k S0 = N, sum_k S1 = sum_n x, sum_k S2 = sum_n x^2 (rows of R sum
    to 1) -- a property that holds at any size."""
    rng = np.random.default_rng(24)
    X, mu, var, lw = _case(rng, 100000, 32, 16, "bf16")
    out = g.gmm_iteration(g.to_device_x(X, "bf16"), mu, var, lw)
    X64 = X.astype(np.float64)
    assert out["S0"].sum() == pytest.approx(100000, rel=TOL_S0_SUM)
    np.testing.assert_allclose(out["S1"].sum(0), X64.sum(0), rtol=1e-5,
                               atol=1e-5 * np.abs(X64).sum(0).max())
    np.testing.assert_allclose(out["S2"].sum(0), (X64 * X64).sum(0), rtol=1e-5)


def test_workload3_prefix(g):
    """Well-separated bf16 mixture (d=32, K=16), first 262144 points."""
    w = WORKLOADS[3]
    X, *_ = gmm_data(w, N=262144)
    mu, var, lw = gmm_init(w, X)
    out = g.gmm_iteration(g.to_device_x(X, "bf16"), mu, var, lw)
    assert out["err"] == 0
    check_gmm_iteration(out, _ref(X, mu, var, lw), "bf16", "w3-prefix")


def test_workload2_prefix_teacher_forced(g):
    """fp32 N=100000 prefix of the d=128, K=256 stream, five EM iterations;
    the oracle takes the GPU's parameters entering each iteration.  Later
    iterations have components that collapse onto single points (variance at
    the floor), which the tensor-core path scores in the direct form."""
    w = WORKLOADS[2]
    X, *_ = gmm_data(w, N=100_000)
    mu, var, lw = gmm_init(w, X)
    Xd = g.to_device_x(X, "f32")
    for it in range(5):
        out = g.gmm_iteration(Xd, mu, var, lw)
        assert out["err"] == 0
        check_gmm_iteration(out, _ref(X, mu, var, lw), "f32", f"w2-prefix-it{it}")
        mu, var, lw = out["means"], out["vars"], out["logw"]


def _n_ill_conditioned(mu, var, bound):
    return int((_cond(mu, var) > bound).sum())


@pytest.mark.slow
def test_workload2_full_size(g):
    """Full N=1,000,000 x 128, K=256 fp32, four teacher-forced EM iterations
    against the oracle (statistics, every point's log-likelihood, updated
    parameters).  Iterations 2-3 are the late-EM state a fit spends its time
    in, with ~15 components collapsed far enough to be scored in the direct
    form."""
    w = WORKLOADS[2]
    X, *_ = gmm_data(w)
    mu, var, lw = gmm_init(w, X)
    Xd = g.to_device_x(X, "f32")
    ws = g.gmm.Workspace.for_gmm(*X.shape, w.K, Xd.dtype)
    for it in range(4):
        out = g.gmm_iteration(Xd, mu, var, lw, ws=ws)
        assert out["err"] == 0, it
        ref = oracle.gmm_em_iteration_onepass(X, mu, var, lw)
        check_gmm_iteration(out, ref, "f32", f"w2-full-it{it}")
        check_stats(out, ref, "f32", f"w2-full-it{it}")
        mu, var, lw = out["means"], out["vars"], out["logw"]
    assert _n_ill_conditioned(mu, var, 2.0 ** 12) > 0


@pytest.mark.slow
def test_workload5_prefix_teacher_forced(g):
    """The large-K bf16 workload (d=128, K=4096, two sweeps) on the first
    200,000 points of its stream, four teacher-forced EM iterations against
    the oracle.  With ~49 points per component EM collapses many components
    within a few iterations, so the later iterations run the direct-form
    kernels with more than 64 listed components (several 16-component passes
    over X); err == 0 at every iteration also shows the slots never run out."""
    w = WORKLOADS[5]
    X, *_ = gmm_data(w, N=200_000)
    mu, var, lw = gmm_init(w, X)
    Xd = g.to_device_x(X, "bf16")
    ws = g.gmm.Workspace.for_gmm(*X.shape, w.K, Xd.dtype)
    from means_clustering_gmm_b200 import _lib
    assert _lib.load().gmm_regime(X.shape[0], w.d, w.K, 1, 0) == 2
    listed = []
    for it in range(4):
        listed.append(_n_ill_conditioned(mu, var, 2.0 ** 12))
        out = g.gmm_iteration(Xd, mu, var, lw, ws=ws)
        assert out["err"] == 0, (it, listed)
        ref = oracle.gmm_em_iteration_onepass(X, mu, var, lw)
        check_gmm_iteration(out, ref, "bf16", f"w5-prefix-it{it}")
        check_stats(out, ref, "bf16", f"w5-prefix-it{it}")
        mu, var, lw = out["means"], out["vars"], out["logw"]
    assert max(listed) > 64, listed


@pytest.mark.slow
def test_workload3_full_size_sampled(g):
    """Full N=16,777,216 bf16: per-point log-likelihood on 4096 sampled points
    (the oracle computes them one by one) and the column-sum identities."""
    w = WORKLOADS[3]
    X, *_ = gmm_data(w)
    mu, var, lw = gmm_init(w, X)
    out = g.gmm_iteration(g.to_device_x(X, "bf16"), mu, var, lw)
    assert out["err"] == 0
    idx = np.random.default_rng(5).choice(X.shape[0], 4096, replace=False)
    ref = oracle.gmm_estep(X[idx], mu, var, lw, want_stats=False)
    assert loglik_err(out["loglik"][idx], ref["loglik"]) <= TOL_LOGLIK
    assert out["S0"].sum() == pytest.approx(X.shape[0], rel=TOL_S0_SUM)
    X64sum = X.astype(np.float64).sum(0)
    np.testing.assert_allclose(out["S1"].sum(0), X64sum, rtol=1e-5, atol=1e-6 * np.abs(X).sum())


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(3000, 64, 5), (4100, 128, 128), (4100, 64, 129),
                                   (6000, 128, 200), (4100, 128, 256), (9000, 128, 300),
                                   (5000, 32, 16), (6000, 32, 200), (9000, 32, 300)])
def test_tensor_core_regimes(g, dtype, shape):
    """Tensor-core kernels: single sweep (one CTA for K <= 128, a cluster of
    two CTAs for K <= 256) and two sweeps (K > 256), each against the oracle;
    the forced two-sweep regime on a single-sweep shape must agree too.
    d = 32 runs zero-padded to one 64-feature block."""
    from means_clustering_gmm_b200 import _lib
    N, d, K = shape
    lib = _lib.load()
    dt = {"f32": 0, "bf16": 1}[dtype]
    assert lib.gmm_regime(N, d, K, dt, 0) == (1 if K <= 256 else 2)
    assert lib.gmm_regime(N, d, K, dt, 1) == 2
    assert lib.gmm_regime(N, d, K, dt, 2) == 0
    rng = np.random.default_rng(N + d + K)
    X, mu, var, lw = _case(rng, N, d, K, dtype)
    Xd = g.to_device_x(X, dtype)
    ref = _ref(X, mu, var, lw)
    out = g.gmm_iteration(Xd, mu, var, lw)
    assert out["err"] == 0
    check_gmm_iteration(out, ref, dtype, f"tc-{shape}-{dtype}")
    check_stats(out, oracle.gmm_estep(X, mu, var, lw), dtype, f"tc-{shape}-{dtype}")
    if K <= 256:
        two = g.gmm_iteration(Xd, mu, var, lw, flags=1)
        assert two["err"] == 0
        check_gmm_iteration(two, ref, dtype, f"tc-two-{shape}-{dtype}")


def _cond(mu, var):
    """Q_k = sum_j mu_kj^2 / var_kj: the size of the terms that cancel in the
    expanded score form x.W1 + x^2.W2 + c for a point near component k."""
    return (mu.astype(np.float64) ** 2 / var.astype(np.float64)).sum(1)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape,flags", [((5000, 128, 100), 0), ((5000, 128, 100), 1),
                                         ((9000, 128, 300), 0), ((4100, 64, 129), 0)])
def test_collapsed_components(g, dtype, shape, flags):
    """Components collapsed onto a data point (mean = the point, variance at or
    near the floor) have Q_k ~ 1e8-1e9: their scores must come out as the
    oracle's (direct form), and a component just below the ill-conditioning
    bound (Q_k ~ 1e4) must still meet the tolerances on the tensor core."""
    N, d, K = shape
    rng = np.random.default_rng(7 * N + K)
    X, mu, var, lw = _case(rng, N, d, K, dtype)
    for k, i, v in [(2, 17, 1e-6), (K // 2, 1000, 1e-6), (K - 1, 4000, 3e-5), (5, 33, 1e-3)]:
        mu[k] = X[i]
        var[k] = v
    q7 = _cond(X[50:51], np.ones((1, d)))[0]
    mu[7] = X[50]
    var[7] = np.float32(q7 / 12000.0)          # Q_7 = 12000, below 2^14
    q = _cond(mu, var)
    assert q[[2, K // 2, K - 1, 5]].min() > 2.0 ** 14 and q[7] < 2.0 ** 14
    ref = _ref(X, mu, var, lw)
    out = g.gmm_iteration(g.to_device_x(X, dtype), mu, var, lw, flags=flags)
    assert out["err"] == 0
    check_gmm_iteration(out, ref, dtype, f"collapsed-{shape}-{dtype}-{flags}")


@pytest.mark.parametrize("shape,nhard", [((12000, 64, 256), 40), ((20000, 64, 2048), 100)])
def test_many_direct_form_components(g, shape, nhard):
    """More ill-conditioned components than one 16-component pass of the
    direct-form scores kernel (K = 256: 40 hard of 64 slots, three passes;
    K = 2048, two-sweep regime: 100 hard of 128 slots, seven passes).  Each
    hard component has Q_k = 3e4 (above 2^14) with a variance that is narrow
    but not degenerate, so its points still carry real responsibility."""
    N, d, K = shape
    rng = np.random.default_rng(11 * N + K)
    X, mu, var, lw = _case(rng, N, d, K, "f32")
    hard = rng.choice(K, size=nhard, replace=False)
    for k in hard:
        q1 = _cond(mu[k:k + 1], np.ones((1, d)))[0]
        var[k] = np.float32(q1 / 3.0e4)
    q = _cond(mu, var)
    assert (q > 2.0 ** 14).sum() >= nhard
    ref = _ref(X, mu, var, lw)
    out = g.gmm_iteration(g.to_device_x(X, "f32"), mu, var, lw)
    assert out["err"] == 0
    check_gmm_iteration(out, ref, "f32", f"many-direct-{shape}")
    assert out["S0"].sum() == pytest.approx(N, rel=TOL_S0_SUM)


def test_too_many_hard_components_reported(g):
    """More hard components than direct-form slots (K = 2048: 128) is reported
    as GMM_ERR_RANGE, not scored silently in the expanded form."""
    N, d, K = 4096, 64, 2048
    rng = np.random.default_rng(5)
    X, mu, var, lw = _case(rng, N, d, K, "f32")
    for k in range(140):
        var[k] = np.float32(_cond(mu[k:k + 1], np.ones((1, d)))[0] / 3.0e4)
    out = g.gmm_iteration(g.to_device_x(X, "f32"), mu, var, lw)
    assert out["err"] == 6   # GMM_ERR_RANGE


@pytest.mark.parametrize("dtype,shape", [("f32", (6000, 64, 40)), ("f32", (5000, 128, 200)),
                                         ("bf16", (9000, 32, 300)), ("f16", (4100, 128, 100))])
def test_uniform_0_1000_data_is_scaled_not_rejected(g, dtype, shape):
    """X ~ U[0, 1000] (far beyond |x| < 181, where x^2 leaves the fp16 range)
    with components as broad as the data (means at data points, variances
    around the data's own): the tensor-core path scales X by 2^-3 and
    matches the oracle with no device error, in all three regimes."""
    N, d, K = shape
    rng = np.random.default_rng(N + K)
    X = round_to(rng.uniform(0, 1000, size=(N, d)).astype(np.float32), dtype)
    mu = X[rng.choice(N, K, replace=False)].astype(np.float32)
    var = (X.astype(np.float64).var(0) * rng.uniform(0.3, 1.5, size=(K, d))).astype(np.float32)
    lw = np.log(rng.dirichlet(np.ones(K))).astype(np.float32)
    from means_clustering_gmm_b200 import _lib
    assert _lib.load().gmm_regime(N, d, K, {"f32": 0, "bf16": 1, "f16": 2}[dtype], 0) in (1, 2)
    out = g.gmm_iteration(g.to_device_x(X, dtype), mu, var, lw)
    assert out["err"] == 0
    check_gmm_iteration(out, _ref(X, mu, var, lw), dtype, f"range-{dtype}-{shape}")
    check_stats(out, oracle.gmm_estep(X, mu, var, lw), dtype, f"range-{dtype}-{shape}")


def test_single_large_value_is_scaled(g):
    """One value of 300 among zeros: scaled, not an error."""
    X = np.zeros((256, 64), np.float32)
    X[3, 5] = 300.0
    mu = np.zeros((4, 64), np.float32)
    mu[1, 5] = 250.0
    var = np.ones((4, 64), np.float32)
    lw = np.full(4, -np.log(4), np.float32)
    out = g.gmm_iteration(g.to_device_x(X, "f32"), mu, var, lw)
    assert out["err"] == 0
    check_gmm_iteration(out, _ref(X, mu, var, lw), "f32", "range-single")


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("N,K", [(1, 1), (127, 5), (129, 16), (5000, 17), (70001, 32),
                                 (300001, 16)])
def test_small_mixture_kernel(g, dtype, N, K):
    """16-bit data, d = 32, K <= 32: the persistent small-mixture kernel
    (E-step hi/lo accumulators, responsibilities in big/small scaled pairs,
    two tile groups in flight), ragged N, K on both sides of 16."""
    d = 32
    rng = np.random.default_rng(N + K)
    X, mu, var, lw = _case(rng, N, d, K, dtype)
    if N >= K:
        mu = X[rng.choice(N, K, replace=False)].astype(np.float32)
    out = g.gmm_iteration(g.to_device_x(X, dtype), mu, var, lw)
    assert out["err"] == 0
    ref = _ref(X, mu, var, lw)
    check_gmm_iteration(out, ref, dtype, f"smallk-{N}-{K}-{dtype}")
    check_stats(out, oracle.gmm_estep(X, mu, var, lw), dtype, f"smallk-{N}-{K}-{dtype}")
    assert out["loglik_total"] == pytest.approx(ref["loglik_total"], rel=1e-6)


def test_small_mixture_kernel_collapsed_and_deterministic(g):
    """Collapsed components (direct form) next to the small-mixture kernel's
    tensor-core components, and bitwise reruns."""
    N, d, K = 40000, 32, 16
    rng = np.random.default_rng(77)
    X, mu, var, lw = _case(rng, N, d, K, "bf16")
    for k, i in [(2, 17), (9, 1000)]:
        mu[k] = X[i]
        var[k] = 1e-6
    Xd = g.to_device_x(X, "bf16")
    a = g.gmm_iteration(Xd, mu, var, lw)
    b = g.gmm_iteration(Xd, mu, var, lw)
    assert a["err"] == 0
    for key in ["means", "vars", "logw", "loglik", "S0", "S1", "S2"]:
        np.testing.assert_array_equal(a[key], b[key])
    check_gmm_iteration(a, _ref(X, mu, var, lw), "bf16", "smallk-collapsed")
