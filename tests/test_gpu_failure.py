"""Failure detection on the GPU without a fault: a bounded wait made to run
out on purpose (GMM_FLAG_TEST_STALL withholds one pipeline stage of the
one-CTA tensor-core kernel) and non-finite inputs.  Each condition must come
back through the workspace's error word, and the next call on the same
workspace must succeed and match the oracle."""
import numpy as np
import pytest
import torch

import means_clustering_gmm_b200 as gmm
import oracle
from means_clustering_gmm_b200 import _lib

from .parity import check_gmm_iteration

pytestmark = pytest.mark.gpu

TIMEOUT, NONFINITE = _lib.GMM_ERR_TIMEOUT, _lib.GMM_ERR_NONFINITE


def _case(seed, N, d, K):
    rng = np.random.default_rng(seed)
    X = (rng.normal(0, 3, size=(K, d))[rng.integers(0, K, N)] +
         rng.standard_normal((N, d))).astype(np.float32)
    mu = X[rng.choice(N, K, replace=False)].copy()
    var = rng.uniform(0.5, 2.0, size=(K, d)).astype(np.float32)
    lw = np.log(rng.dirichlet(np.ones(K))).astype(np.float32)
    return X, mu, var, lw


def _dev(*a):
    return [torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in a]


@pytest.mark.parametrize("flags", [0, 1])   # one-CTA single sweep; sweep 1 of two sweeps
def test_bounded_wait_runs_out_then_workspace_recovers(flags):
    N, d, K = 6000, 64, 100 if flags == 0 else 200
    X, mu, var, lw = _case(50 + flags, N, d, K)
    Xd, m, v, l = _dev(X, mu, var, lw)
    ws = gmm.Workspace.for_gmm(N, d, K)
    gmm.gmm_em_step(Xd, m, v, l, ws, flags=flags | _lib.GMM_FLAG_TEST_STALL)
    assert gmm.gmm_last_error(ws) == TIMEOUT
    # the context and the workspace are still usable: the same call again
    from . import gpu_helpers
    out = gpu_helpers.gmm_iteration(Xd, mu, var, lw, flags=flags, ws=ws)
    assert out["err"] == 0
    check_gmm_iteration(out, oracle.gmm_em_iteration(X, mu, var, lw), "f32",
                        f"after-timeout-{flags}")


@pytest.mark.parametrize("d,flags", [(64, 0), (16, 0), (64, 2)])
def test_nonfinite_parameters_reported(d, flags):
    """A NaN variance, an infinite mean and a NaN log weight, on the
    tensor-core (d = 64) and CUDA-core (d = 16, or FORCE_SIMT) paths."""
    N, K = 3000, 20
    X, mu, var, lw = _case(60 + d, N, d, K)
    Xd = _dev(X)[0]
    ws = gmm.Workspace.for_gmm(N, d, K)
    for name in ("var", "mu", "logw"):
        m, v, l = (a.copy() for a in (mu, var, lw))
        if name == "var":
            v[3, 2] = np.nan
        elif name == "mu":
            m[5, 1] = np.inf
        else:
            l[7] = np.nan
        mt, vt, lt = _dev(m, v, l)
        gmm.gmm_em_step(Xd, mt, vt, lt, ws, flags=flags)
        assert gmm.gmm_last_error(ws) == NONFINITE, name
    from . import gpu_helpers
    out = gpu_helpers.gmm_iteration(Xd, mu, var, lw, flags=flags, ws=ws)
    assert out["err"] == 0
    check_gmm_iteration(out, oracle.gmm_em_iteration(X, mu, var, lw), "f32", f"after-nan-{d}")


def test_nan_in_the_data_reported_by_the_finalise():
    """A NaN feature value makes that point's responsibilities NaN, so the
    M-step finalise meets non-finite statistics and reports them."""
    N, d, K = 4000, 64, 30
    X, mu, var, lw = _case(70, N, d, K)
    Xbad = X.copy()
    Xbad[123, 4] = np.nan
    Xd, m, v, l = _dev(Xbad, mu, var, lw)
    ws = gmm.Workspace.for_gmm(N, d, K)
    stats, _, _ = gmm.gmm_em_step(Xd, m, v, l, ws)
    gmm.gmm_finalize(stats, N, m, v, l, ws)
    assert gmm.gmm_last_error(ws) == NONFINITE


def test_checkpoint_resume_is_bitwise():
    """The EM state is (means, vars, log w): save it after 3 iterations,
    reload it into fresh buffers and run 3 more; the result equals 6
    uninterrupted iterations bit for bit (the kernels are deterministic)."""
    N, d, K = 20000, 128, 64
    X, mu, var, lw = _case(80, N, d, K)
    Xd = _dev(X)[0]
    ws = gmm.Workspace.for_gmm(N, d, K)
    m, v, l = _dev(mu, var, lw)
    for _ in range(6):
        gmm.em_iteration(Xd, m, v, l, ws)
    straight = [t.cpu().numpy() for t in (m, v, l)]
    m, v, l = _dev(mu, var, lw)
    for _ in range(3):
        gmm.em_iteration(Xd, m, v, l, ws)
    saved = [t.cpu().numpy().copy() for t in (m, v, l)]   # checkpoint
    m, v, l = _dev(*saved)                                 # resume
    ws2 = gmm.Workspace.for_gmm(N, d, K)
    for _ in range(3):
        gmm.em_iteration(Xd, m, v, l, ws2)
    assert gmm.gmm_last_error(ws) == 0 and gmm.gmm_last_error(ws2) == 0
    for a, b in zip(straight, (m, v, l)):
        np.testing.assert_array_equal(a, b.cpu().numpy())
