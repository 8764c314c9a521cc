"""Pins for the float64 oracle: closed forms, invariants, brute force and a
library special case -- never the oracle against itself.

Each test is chosen so that a plausible slip in the oracle (a dropped
log-variance term, a sign, a swapped index, a missing renormalisation, a
one-pass variance) fails at least one of them.
"""
import math
import warnings

import numpy as np
import pytest

import oracle
from oracle import brute
from synth import WORKLOADS, gmm_data, gmm_init

pytestmark = pytest.mark.usefixtures("oracle_lib")


def _rand_params(rng, K, d, spread=3.0):
    mu = rng.normal(0, spread, size=(K, d))
    var = rng.uniform(0.2, 2.0, size=(K, d))
    w = rng.dirichlet(np.ones(K))
    return mu, var, w


def test_log_density_matches_scipy_closed_form():
    """K=1, weight 1: l_n is the sum over dimensions of the univariate normal
    log-pdf (library routine scipy.stats.norm.logpdf)."""
    from scipy.stats import norm
    rng = np.random.default_rng(1)
    X = rng.normal(0, 2, size=(50, 5))
    mu = rng.normal(0, 1, size=(1, 5))
    var = rng.uniform(0.3, 3.0, size=(1, 5))
    out = oracle.gmm_estep(X, mu, var, np.zeros(1))
    ref = norm.logpdf(X, loc=mu[0], scale=np.sqrt(var[0])).sum(axis=1)
    np.testing.assert_allclose(out["loglik"], ref, rtol=1e-13, atol=1e-12)
    assert out["loglik_total"] == pytest.approx(ref.sum(), rel=1e-13)


def test_k1_gives_sample_mean_and_population_variance():
    """K=1: responsibilities are all 1, so one EM step returns the sample mean,
    the population variance (divisor N) and weight 1."""
    rng = np.random.default_rng(2)
    X = rng.normal(3, 1.7, size=(1000, 7))
    out = oracle.gmm_em_iteration(X, rng.normal(size=(1, 7)), np.ones((1, 7)), np.zeros(1),
                                  var_floor=0.0)
    np.testing.assert_allclose(out["means"][0], X.mean(axis=0), rtol=1e-13)
    np.testing.assert_allclose(out["vars"][0], X.var(axis=0), rtol=1e-12)
    assert out["logw"][0] == pytest.approx(0.0, abs=1e-15)
    assert out["Nk"][0] == pytest.approx(1000.0, rel=1e-14)


def test_brute_force_tiny():
    """N=7, d=3, K=4 against the pure-Python brute force (direct exp, fsum)."""
    rng = np.random.default_rng(3)
    X = rng.normal(0, 1.5, size=(7, 3))
    mu, var, w = _rand_params(rng, 4, 3, spread=1.0)
    R_b, ll_b = brute.responsibilities(X.tolist(), mu.tolist(), var.tolist(), w.tolist())
    out = oracle.gmm_estep(X, mu, var, np.log(w), want_R=True)
    np.testing.assert_allclose(out["R"], np.array(R_b), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(out["loglik"], np.array(ll_b), rtol=1e-13)
    m_b, v_b, w_b, L_b = brute.em_iteration(X.tolist(), mu.tolist(), var.tolist(), w.tolist())
    it = oracle.gmm_em_iteration(X, mu, var, np.log(w), var_floor=0.0)
    np.testing.assert_allclose(it["means"], np.array(m_b), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(it["vars"], np.array(v_b), rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(np.exp(it["logw"]), np.array(w_b), rtol=1e-12)
    assert it["loglik_total"] == pytest.approx(L_b, rel=1e-13)


def test_raw_statistics_match_definition_tiny():
    """S0 | S1 | S2 are sum r, sum r x, sum r x^2 with the brute-force R."""
    rng = np.random.default_rng(4)
    X = rng.normal(0, 1.0, size=(6, 2))
    mu, var, w = _rand_params(rng, 3, 2, spread=0.8)
    R_b, _ = brute.responsibilities(X.tolist(), mu.tolist(), var.tolist(), w.tolist())
    R_b = np.array(R_b)
    out = oracle.gmm_estep(X, mu, var, np.log(w))
    np.testing.assert_allclose(out["S0"], R_b.sum(axis=0), rtol=1e-12)
    np.testing.assert_allclose(out["S1"], R_b.T @ X, rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(out["S2"], R_b.T @ (X * X), rtol=1e-11, atol=1e-14)


def test_rows_sum_to_one_and_stats_column_sums():
    """Each row of R sums to 1, hence sum_k S0 = N, sum_k S1 = sum_n x_n and
    sum_k S2 = sum_n x_n^2 (exact identities in real arithmetic)."""
    rng = np.random.default_rng(5)
    X = rng.normal(0, 3, size=(3000, 6))
    mu, var, w = _rand_params(rng, 16, 6)
    out = oracle.gmm_estep(X, mu, var, np.log(w), want_R=True)
    np.testing.assert_allclose(out["R"].sum(axis=1), 1.0, atol=1e-12)
    assert out["S0"].sum() == pytest.approx(3000.0, rel=1e-12)
    np.testing.assert_allclose(out["S1"].sum(axis=0), X.sum(axis=0), rtol=1e-10, atol=1e-9)
    np.testing.assert_allclose(out["S2"].sum(axis=0), (X * X).sum(axis=0), rtol=1e-12)


def test_component_permutation_permutes_outputs():
    rng = np.random.default_rng(6)
    X = rng.normal(0, 2, size=(500, 4))
    mu, var, w = _rand_params(rng, 5, 4)
    perm = rng.permutation(5)
    a = oracle.gmm_estep(X, mu, var, np.log(w), want_R=True)
    b = oracle.gmm_estep(X, mu[perm], var[perm], np.log(w)[perm], want_R=True)
    np.testing.assert_allclose(b["R"], a["R"][:, perm], rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(b["loglik"], a["loglik"], rtol=1e-13)
    np.testing.assert_allclose(b["S1"], a["S1"][perm], rtol=1e-11, atol=1e-12)


def test_common_shift_leaves_responsibilities_unchanged():
    """Shifting X and every mean by the same vector changes nothing."""
    rng = np.random.default_rng(7)
    X = rng.normal(0, 2, size=(400, 3))
    mu, var, w = _rand_params(rng, 4, 3)
    c = np.array([10.0, -3.0, 0.5])
    a = oracle.gmm_estep(X, mu, var, np.log(w), want_R=True)
    b = oracle.gmm_estep(X + c, mu + c, var, np.log(w), want_R=True)
    np.testing.assert_allclose(b["R"], a["R"], rtol=1e-9, atol=1e-14)
    np.testing.assert_allclose(b["loglik"], a["loglik"], rtol=1e-11)


def test_sklearn_diag_mstep_special_case():
    """One EM step from given parameters equals scikit-learn's diagonal
    GaussianMixture (reg_covar=0, one iteration from the same initial state)."""
    from sklearn.exceptions import ConvergenceWarning
    from sklearn.mixture import GaussianMixture
    rng = np.random.default_rng(8)
    X = rng.normal(0, 2, size=(300, 4))
    mu, var, w = _rand_params(rng, 3, 4, spread=1.5)
    gm = GaussianMixture(n_components=3, covariance_type="diag", reg_covar=0.0, max_iter=1,
                         n_init=1, tol=0.0, weights_init=w, means_init=mu,
                         precisions_init=1.0 / var, random_state=0)
    with warnings.catch_warnings():
        warnings.simplefilter("ignore", ConvergenceWarning)
        gm.fit(X)
    it = oracle.gmm_em_iteration(X, mu, var, np.log(w), var_floor=0.0)
    np.testing.assert_allclose(it["means"], gm.means_, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(it["vars"], gm.covariances_, rtol=1e-8, atol=1e-11)
    np.testing.assert_allclose(np.exp(it["logw"]), gm.weights_, rtol=1e-10)


def test_two_point_closed_form():
    """Hand-derived: x = {-1, +1}, K=2 with means -1/+1, unit variance, equal
    weights: r = 1/(1+e^-2) for the own component; one EM step moves each mean
    to (r*x_own + (1-r)*x_other)."""
    X = np.array([[-1.0], [1.0]])
    out = oracle.gmm_em_iteration(X, np.array([[-1.0], [1.0]]), np.ones((2, 1)),
                                  np.log([0.5, 0.5]), var_floor=0.0)
    r = 1.0 / (1.0 + math.exp(-2.0))
    m0 = (r * -1.0 + (1 - r) * 1.0) / 1.0
    assert out["means"][0, 0] == pytest.approx(m0, rel=1e-14)
    assert out["means"][1, 0] == pytest.approx(-m0, rel=1e-14)
    v0 = r * (-1.0 - m0) ** 2 + (1 - r) * (1.0 - m0) ** 2
    assert out["vars"][0, 0] == pytest.approx(v0, rel=1e-13)
    l1 = math.log(0.5 * math.exp(-0.5 * math.log(2 * math.pi))
                  + 0.5 * math.exp(-0.5 * math.log(2 * math.pi) - 2.0))
    np.testing.assert_allclose(out["loglik"], [l1, l1], rtol=1e-14)


def test_golden_hand_examples():
    """Worked examples derived by hand from the definitions (tests/golden)."""
    import json
    import os
    from fractions import Fraction
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_em_hand.json")
    with open(path) as f:
        cases = json.load(f)["cases"]
    frac = np.vectorize(lambda s: float(Fraction(s)))
    for c in cases:
        it = oracle.gmm_em_iteration(np.array(c["X"]), np.array(c["means"]),
                                     np.array(c["vars"]), np.log(np.array(c["weights"])),
                                     var_floor=0.0)
        np.testing.assert_allclose(it["means"], frac(np.array(c["expect_means"])), rtol=1e-14)
        np.testing.assert_allclose(it["vars"], frac(np.array(c["expect_vars"])), rtol=1e-14)
        exp_ll = [float(Fraction(q)) - 0.5 * n2pi * math.log(2 * math.pi)
                  - 0.5 * sum(math.log(v) for v in lv)
                  for q, n2pi, lv in c["expect_loglik"]]
        np.testing.assert_allclose(it["loglik"], exp_ll, rtol=1e-14)


def test_loglik_never_decreases_small_workload():
    """EM monotonicity on the 4096 x 16, K=8 workload for 10 iterations."""
    w = WORKLOADS[1]
    X, *_ = gmm_data(w)
    mu, var, lw = gmm_init(w, X)
    L = []
    for _ in range(10):
        it = oracle.gmm_em_iteration(X, mu, var, lw)
        L.append(it["loglik_total"])
        mu, var, lw = it["means"], it["vars"], it["logw"]
    for a, b in zip(L, L[1:]):
        assert b >= a - 1e-12 * abs(a)


def test_loglik_never_decreases_medium_workload():
    """Same invariant on a prefix of the N=1M, d=128, K=256 stream, reduced to
    20000 points and the first 32 dimensions / 32 components."""
    w = WORKLOADS[2]
    X, *_ = gmm_data(w, N=20000)
    X = X[:, :32]
    mu, var, lw = gmm_init(w, X, K=32)
    L = []
    for _ in range(10):
        it = oracle.gmm_em_iteration(X, mu, var, lw)
        L.append(it["loglik_total"])
        mu, var, lw = it["means"], it["vars"], it["logw"]
    for a, b in zip(L, L[1:]):
        assert b >= a - 1e-12 * abs(a)


def test_recovers_well_separated_parameters():
    """Well-separated mixture (means ~ U[-8,8]^32, sigma 1, Dirichlet(2)
    weights), initialised with one point per true component: after 20
    iterations |mu_hat - mu| <= 5 sigma / sqrt(N_k) and
    |w_hat - w| <= 5 sqrt(w (1-w) / N)."""
    w = WORKLOADS[3]
    N = 200_000
    X, labels, mu_t, sig_t, w_t = gmm_data(w, N=N)
    rng = np.random.default_rng(99)
    first = np.array([rng.choice(np.flatnonzero(labels == k)) for k in range(w.K)])
    mu = X[first].astype(np.float64)
    var = np.ones_like(mu)
    lw = np.full(w.K, -math.log(w.K))
    for _ in range(20):
        it = oracle.gmm_em_iteration(X, mu, var, lw)
        mu, var, lw = it["means"], it["vars"], it["logw"]
    Nk = np.exp(lw) * N
    bound = 5.0 * sig_t / np.sqrt(Nk)[:, None]
    assert np.all(np.abs(mu - mu_t) <= bound)
    wb = 5.0 * np.sqrt(w_t * (1 - w_t) / N)
    assert np.all(np.abs(np.exp(lw) - w_t) <= wb)


def test_degenerate_component_keeps_parameters():
    """A zero-weight component (log w = -inf) gets N_k = 0: it keeps its mean
    and variance and its log weight stays -inf."""
    rng = np.random.default_rng(10)
    X = rng.normal(0, 1, size=(100, 2))
    mu = np.array([[0.0, 0.0], [50.0, 50.0]])
    var = np.array([[1.0, 1.0], [2.0, 3.0]])
    it = oracle.gmm_em_iteration(X, mu, var, np.array([0.0, -np.inf]), var_floor=0.0)
    np.testing.assert_array_equal(it["means"][1], mu[1])
    np.testing.assert_array_equal(it["vars"][1], var[1])
    assert it["logw"][1] == -np.inf
    np.testing.assert_allclose(it["means"][0], X.mean(axis=0), rtol=1e-12)


def test_variance_floor_clamps():
    X = np.array([[1.0], [1.0], [1.0]])
    it = oracle.gmm_em_iteration(X, np.array([[0.0]]), np.array([[1.0]]), np.zeros(1),
                                 var_floor=1e-6)
    assert it["vars"][0, 0] == 1e-6


# ---------------------------------------------------------------- k-means

def test_lloyd_brute_force_tiny():
    rng = np.random.default_rng(11)
    X = rng.normal(0, 1, size=(9, 3))
    C = rng.normal(0, 1, size=(4, 3))
    ids_b, C_b = brute.lloyd(X.tolist(), C.tolist())
    out = oracle.kmeans_step(X[None], C[None])
    np.testing.assert_array_equal(out["ids"][0], ids_b)
    np.testing.assert_allclose(out["centroids"][0], np.array(C_b), rtol=1e-14)


def test_lloyd_numpy_argmin_and_member_means():
    """N=4096: ids equal numpy's argmin of the full distance matrix; each new
    centroid is the numpy mean of its members; inertia is the sum of minima."""
    rng = np.random.default_rng(12)
    X = rng.normal(0, 1, size=(2, 4096, 16))
    C = rng.normal(0, 1, size=(2, 64, 16))
    out = oracle.kmeans_step(X, C)
    for b in range(2):
        D = ((X[b][:, None, :] - C[b][None, :, :]) ** 2).sum(-1)
        np.testing.assert_array_equal(out["ids"][b], D.argmin(axis=1))
        assert out["inertia"][b] == pytest.approx(D.min(axis=1).sum(), rel=1e-12)
        srt = np.sort(D, axis=1)
        np.testing.assert_allclose(out["d1"][b], srt[:, 0], rtol=1e-12)
        np.testing.assert_allclose(out["d2"][b], srt[:, 1], rtol=1e-12)
        for k in range(64):
            m = out["ids"][b] == k
            exp = X[b][m].mean(axis=0) if m.any() else C[b][k]
            np.testing.assert_allclose(out["centroids"][b][k], exp, rtol=1e-12, atol=1e-14)
            assert out["counts"][b][k] == m.sum()


def test_lloyd_ties_go_to_lowest_index_and_empty_keeps_old():
    X = np.array([[[0.0, 0.0], [4.0, 0.0]]])
    C = np.array([[[-1.0, 0.0], [1.0, 0.0], [9.0, 9.0], [5.0, 0.0]]])
    out = oracle.kmeans_step(X, C)
    # point 0 is exactly 1 away from centroids 0 and 1 -> centroid 0
    assert out["ids"][0, 0] == 0
    # point 1 is 3 from centroid 1 and 1 from centroid 3 -> centroid 3
    assert out["ids"][0, 1] == 3
    np.testing.assert_array_equal(out["centroids"][0, 1], C[0, 1])   # empty: kept
    np.testing.assert_array_equal(out["centroids"][0, 2], C[0, 2])   # empty: kept


def test_lloyd_inertia_non_increasing():
    rng = np.random.default_rng(13)
    X = rng.normal(0, 1, size=(1, 3000, 8))
    C = X[:, rng.choice(3000, 32, replace=False)]
    prev = np.inf
    for _ in range(8):
        out = oracle.kmeans_step(X, C)
        assert out["inertia"][0] <= prev * (1 + 1e-12)
        prev = out["inertia"][0]
        C = out["centroids"]


def test_kmeans_update_is_member_mean():
    """Teacher-forced update: numpy mean of the members for arbitrary ids."""
    rng = np.random.default_rng(14)
    X = rng.normal(0, 1, size=(2, 500, 5))
    C = rng.normal(0, 1, size=(2, 9, 5))
    ids = rng.integers(0, 8, size=(2, 500)).astype(np.int32)   # cluster 8 stays empty
    Co, cnt = oracle.kmeans_update(X, ids, C)
    for b in range(2):
        for k in range(9):
            m = ids[b] == k
            exp = X[b][m].mean(axis=0) if m.any() else C[b][k]
            np.testing.assert_allclose(Co[b][k], exp, rtol=1e-13, atol=1e-15)
            assert cnt[b][k] == m.sum()


# ------------------------------------------- one-pass M-step from statistics

def test_mstep_from_stats_k1_closed_form():
    """K=1: the M-step from the statistics of one E-step is the sample mean
    and the population variance (numpy), weight 1."""
    rng = np.random.default_rng(31)
    X = rng.normal(-2, 0.7, size=(777, 5))
    e = oracle.gmm_estep(X, rng.normal(size=(1, 5)), np.ones((1, 5)), np.zeros(1))
    m = oracle.gmm_mstep(e["stats"], 777, np.zeros((1, 5)), np.ones((1, 5)), var_floor=0.0)
    np.testing.assert_allclose(m["means"][0], X.mean(axis=0), rtol=1e-13)
    np.testing.assert_allclose(m["vars"][0], X.var(axis=0), rtol=1e-11)
    assert m["logw"][0] == pytest.approx(0.0, abs=1e-15)


def test_mstep_from_stats_matches_sklearn():
    """The one-pass iteration (estep + mstep) reproduces scikit-learn's
    diagonal GaussianMixture step (reg_covar=0) on a 3-component mixture."""
    from sklearn.exceptions import ConvergenceWarning
    from sklearn.mixture import GaussianMixture
    rng = np.random.default_rng(32)
    X = rng.normal(0, 2, size=(400, 3))
    mu, var, w = _rand_params(rng, 3, 3, spread=1.5)
    gm = GaussianMixture(n_components=3, covariance_type="diag", reg_covar=0.0, max_iter=1,
                         n_init=1, tol=0.0, weights_init=w, means_init=mu,
                         precisions_init=1.0 / var, random_state=0)
    with warnings.catch_warnings():
        warnings.simplefilter("ignore", ConvergenceWarning)
        gm.fit(X)
    it = oracle.gmm_em_iteration_onepass(X, mu, var, np.log(w), var_floor=0.0)
    np.testing.assert_allclose(it["means"], gm.means_, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(it["vars"], gm.covariances_, rtol=1e-8, atol=1e-11)
    np.testing.assert_allclose(np.exp(it["logw"]), gm.weights_, rtol=1e-10)


def test_mstep_from_stats_degenerate_and_floor():
    """A zero-mass component keeps its parameters and gets log w = -inf; a
    zero-variance feature is clamped at the floor."""
    X = np.array([[1.0, 0.0], [1.0, 2.0], [1.0, 4.0]])
    mu = np.array([[0.0, 0.0], [50.0, 50.0]])
    var = np.array([[1.0, 1.0], [2.0, 3.0]])
    it = oracle.gmm_em_iteration_onepass(X, mu, var, np.array([0.0, -np.inf]), var_floor=1e-6)
    np.testing.assert_array_equal(it["means"][1], mu[1])
    np.testing.assert_array_equal(it["vars"][1], var[1])
    assert it["logw"][1] == -np.inf
    assert it["vars"][0, 0] == 1e-6
    assert it["vars"][0, 1] == pytest.approx(8.0 / 3.0, rel=1e-14)
    np.testing.assert_allclose(it["means"][0], [1.0, 2.0], rtol=1e-15)


def test_hard_mstep_is_per_cluster_mean_and_variance():
    """The M-step of a hard partition: per-cluster numpy mean and population
    variance; an empty cluster keeps its centroid with variance 1; weights
    max(n_k, 1) / (N + empty)."""
    rng = np.random.default_rng(33)
    N, d, K = 500, 4, 5
    X = rng.normal(0, 3, size=(N, d))
    ids = rng.integers(0, K - 1, size=N).astype(np.int32)   # cluster K-1 stays empty
    ids[:3] = 0
    C = rng.normal(size=(K, d))
    out = oracle.gmm_hard_mstep(X, ids, C, var_floor=1e-9)
    for k in range(K - 1):
        m = ids == k
        np.testing.assert_allclose(out["means"][k], X[m].mean(axis=0), rtol=1e-13)
        np.testing.assert_allclose(out["vars"][k], X[m].var(axis=0), rtol=1e-12)
        assert out["logw"][k] == pytest.approx(math.log(m.sum() / (N + 1)), rel=1e-14)
    np.testing.assert_array_equal(out["means"][K - 1], C[K - 1])
    np.testing.assert_array_equal(out["vars"][K - 1], np.ones(d))
    assert out["logw"][K - 1] == pytest.approx(math.log(1.0 / (N + 1)), rel=1e-14)
    # a single-member cluster's variance is clamped at the floor
    ids2 = np.zeros(N, np.int32)
    ids2[7] = 1
    out2 = oracle.gmm_hard_mstep(X, ids2, C[:2], var_floor=0.25)
    np.testing.assert_array_equal(out2["vars"][1], np.full(d, 0.25))
