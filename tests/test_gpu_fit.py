"""The on-device EM fit loop (gmm_fit) and the k-means start of a fit
(gmm_init_kmeans), through the C ABI, against the float64 oracle.

gmm_fit runs gmm_em_step + gmm_finalize inside one CUDA graph with a
conditional WHILE node; the loop must run the same kernels as a host loop
(bitwise equal results after the same number of iterations), stop on the
device-side test |L_t - L_{t-1}| <= tol |L_t|, never let L decrease beyond
rounding, and end at a point the oracle agrees is an EM fixed point."""
import numpy as np
import pytest
import torch

import means_clustering_gmm_b200 as gmm
import oracle
from synth import WORKLOADS, gmm_data, gmm_init, round_to

from .parity import check_gmm_iteration, normwise

pytestmark = pytest.mark.gpu


def _dev(*arrays):
    return [torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda() for a in arrays]


def _host_loop(Xd, mu, var, lw, iters, flags=0):
    """The same EM iterations issued from the host, one call pair each."""
    m, v, l = _dev(mu, var, lw)
    ws = gmm.Workspace.for_gmm(Xd.shape[0], Xd.shape[1], m.shape[0], Xd.dtype)
    for _ in range(iters):
        gmm.em_iteration(Xd, m, v, l, ws, flags=flags)
    assert gmm.gmm_last_error(ws) == 0
    return m.cpu().numpy(), v.cpu().numpy(), l.cpu().numpy()


def _monotone(trace):
    tr = np.asarray(trace, np.float64)
    # EM never decreases L in exact arithmetic; allow fp32 rounding of the
    # per-point terms near convergence
    return bool(np.all(np.diff(tr) >= -1e-6 * np.abs(tr[1:])))


def _fixed_point_check(X, dtype, m, v, l, label):
    """One more iteration from the fitted parameters, teacher-forced against
    the oracle; at convergence it barely moves them."""
    from . import gpu_helpers
    Xd = gpu_helpers.to_device_x(X, dtype)
    nxt = gpu_helpers.gmm_iteration(Xd, m, v, l)
    assert nxt["err"] == 0
    ref = oracle.gmm_em_iteration(X, m, v, l)
    check_gmm_iteration(nxt, ref, dtype, label)
    return nxt


def test_fit_workload1_converges():
    """4096 x 16, K = 8 (fp32): the loop converges on the device, L is
    monotone, the result equals a host loop of the same length bit for bit,
    and it is an EM fixed point per the oracle."""
    w = WORKLOADS[1]
    X, *_ = gmm_data(w)
    mu, var, lw = gmm_init(w, X)
    Xd = torch.from_numpy(X).cuda()
    m0, v0, l0 = _dev(mu, var, lw)
    m, v, l, trace, conv = gmm.fit(Xd, m0, v0, l0, max_iters=500, tol=1e-8)
    tr = trace.cpu().numpy()
    assert conv, len(tr)
    assert 2 <= len(tr) < 500
    assert _monotone(tr), np.diff(tr).min()
    assert tr[-1] > tr[0]
    hm, hv, hl = _host_loop(Xd, mu, var, lw, len(tr))
    np.testing.assert_array_equal(m.cpu().numpy(), hm)
    np.testing.assert_array_equal(v.cpu().numpy(), hv)
    np.testing.assert_array_equal(l.cpu().numpy(), hl)
    mf, vf, lf = m.cpu().numpy(), v.cpu().numpy(), l.cpu().numpy()
    nxt = _fixed_point_check(X, "f32", mf, vf, lf, "fit-w1-fixed-point")
    # |dL| <= tol |L| still lets parameters move in flat directions (L is
    # quadratic in them near the optimum): a small step, not none
    assert normwise(nxt["means"], mf) <= 1e-3
    # L at the fitted parameters (oracle) is within the tolerance of the last
    # L the loop computed (at the parameters one M-step earlier)
    ref_L = oracle.gmm_estep(X, mf, vf, lf, want_stats=False)["loglik_total"]
    assert abs(ref_L - tr[-1]) <= 1e-6 * abs(tr[-1])


def test_fit_workload2_prefix_and_api_host_tensors():
    """The first 50,000 points of the N=1M, d=128, K=256 fp32 workload (the
    tcgen05 cluster kernel, components collapsing into the direct form):
    30 iterations at most, through api.fit with host tensors (copied in and
    out); monotone L, bitwise equal to the host loop, and a teacher-forced
    oracle check at the end."""
    w = WORKLOADS[2]
    X, *_ = gmm_data(w, N=50_000)
    mu, var, lw = gmm_init(w, X)
    m, v, l, trace, conv = gmm.fit(torch.from_numpy(X), torch.from_numpy(mu),
                                   torch.from_numpy(var), torch.from_numpy(lw),
                                   max_iters=30, tol=1e-7)
    assert not m.is_cuda
    tr = trace.numpy()
    assert 2 <= len(tr) <= 30 and (conv or len(tr) == 30)
    assert _monotone(tr), np.diff(tr).min()
    Xd = torch.from_numpy(X).cuda()
    hm, hv, hl = _host_loop(Xd, mu, var, lw, len(tr))
    np.testing.assert_array_equal(m.numpy(), hm)
    np.testing.assert_array_equal(v.numpy(), hv)
    np.testing.assert_array_equal(l.numpy(), hl)
    _fixed_point_check(X, "f32", m.numpy(), v.numpy(), l.numpy(), "fit-w2-prefix-last")


def test_fit_stops_at_max_iters_and_reports():
    """tol = 0 never passes unless L repeats exactly: the loop runs max_iters
    iterations and reports not converged; the trace holds every L_t."""
    rng = np.random.default_rng(40)
    N, d, K = 3000, 32, 12
    X = rng.normal(0, 3, size=(N, d)).astype(np.float32)
    mu = X[rng.choice(N, K, replace=False)]
    var = np.ones((K, d), np.float32)
    lw = np.full(K, -np.log(K), np.float32)
    Xd = torch.from_numpy(X).cuda()
    m0, v0, l0 = _dev(mu, var, lw)
    m, v, l, trace, conv = gmm.fit(Xd, m0, v0, l0, max_iters=3, tol=0.0)
    assert len(trace) == 3 and not conv
    ref = oracle.gmm_estep(X, mu, var, lw, want_stats=False)
    assert trace[0].item() == pytest.approx(ref["loglik_total"], rel=1e-6)
    hm, hv, hl = _host_loop(Xd, mu, var, lw, 3)
    np.testing.assert_array_equal(m.cpu().numpy(), hm)


def _blobs(seed, N, d, K, spread=4.0, sigma=0.1):
    rng = np.random.default_rng(seed)
    centres = rng.normal(0, spread, size=(K, d))
    lab = rng.integers(0, K, size=N)
    X = (centres[lab] + sigma * rng.standard_normal((N, d))).astype(np.float32)
    return X, rng


@pytest.mark.parametrize("dtype,d", [("f32", 64), ("f16", 128), ("bf16", 40)])
@pytest.mark.parametrize("iters", [1, 5])
def test_init_kmeans_matches_oracle(dtype, d, iters):
    """gmm_init_kmeans: `iters` Lloyd iterations, then the hard partition's
    M-step.  With one iteration the ids equal the oracle's assignment
    (except near-ties); after five, Lloyd trajectories may part at points
    between two centroids of one split blob, so the ids are checked for broad
    agreement and the parameters teacher-forced: means, variances and weights
    equal the oracle's hard M-step of the GPU's own partition."""
    N, K = 20000, 48
    X, rng = _blobs(7 + d, N, d, K)
    X = round_to(X, dtype)
    C0 = X[np.sort(rng.choice(N, K, replace=False))].copy()
    from . import gpu_helpers
    Xd = gpu_helpers.to_device_x(X, dtype)
    m, v, l, ids = gmm.init_kmeans(Xd, torch.from_numpy(C0).cuda(), iters=iters, want_ids=True)
    torch.cuda.synchronize()
    ids = ids.cpu().numpy()
    C = C0.astype(np.float64)
    for _ in range(iters):
        step = oracle.kmeans_step(X, C)
        C = step["centroids"][0]
    differ = ids != step["ids"][0]
    if iters == 1:
        gap = (step["d2"][0] - step["d1"][0]) / np.where(step["d1"][0] > 0, step["d1"][0], 1)
        tie = (step["d1"][0] > 0) & (gap < 1e-3)
        assert not (differ & ~tie).any()
    else:
        assert differ.mean() < 0.05, differ.mean()
    # (an empty cluster keeps the centroid of its own trajectory: compared by
    # weight only)
    ref = oracle.gmm_hard_mstep(X, ids, C0)
    got = {"means": m.cpu().numpy(), "vars": v.cpu().numpy(), "logw": l.cpu().numpy()}
    counts = np.bincount(ids, minlength=K)
    live = counts > 0
    check_gmm_iteration({k: a[live] for k, a in got.items()},
                        {k: a[live] for k, a in ref.items()}, dtype,
                        f"init-kmeans-{dtype}-{d}-{iters}")
    np.testing.assert_allclose(got["logw"], ref["logw"], rtol=1e-6)


def test_fit_from_kmeans_start():
    """The usual pipeline: k-means start, then the EM fit, on well-separated
    blobs: the fit converges and recovers one component per blob."""
    N, d, K = 30000, 64, 16
    X, rng = _blobs(99, N, d, K, spread=3.0, sigma=0.3)
    Xd = torch.from_numpy(X).cuda()
    C0 = torch.from_numpy(X[np.sort(rng.choice(N, K, replace=False))].copy()).cuda()
    m, v, l = gmm.init_kmeans(Xd, C0, iters=10)
    m, v, l, trace, conv = gmm.fit(Xd, m, v, l, max_iters=300, tol=1e-6)
    assert _monotone(trace.cpu().numpy())
    assert conv, len(trace)
    _fixed_point_check(X, "f32", m.cpu().numpy(), v.cpu().numpy(), l.cpu().numpy(),
                       "fit-from-kmeans")
