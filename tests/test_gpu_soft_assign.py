"""Soft multi-assignment (gmm_soft_assign): per point the top-r components by
responsibility with r_nk >= tau, against the oracle's explicit N x K
responsibility matrix.  Where floating point decides the selection (two
responsibilities, or one and tau, closer than the tolerance), any valid
choice is accepted; everywhere else the selected ids must be the oracle's."""
import numpy as np
import pytest
import torch

import means_clustering_gmm_b200 as gmm
import oracle
from synth import round_to

from .parity import TOL_LOGLIK, loglik_err

pytestmark = pytest.mark.gpu
TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}
TOL_R = 1e-3   # absolute, on responsibilities in [0, 1]


def _case(seed, N, d, K, dtype, spread=1.2):
    rng = np.random.default_rng(seed)
    centres = rng.normal(0, spread, size=(K, d))
    X = round_to((centres[rng.integers(0, K, N)] +
                  rng.standard_normal((N, d))).astype(np.float32), dtype)
    mu = X[rng.choice(N, K, replace=False)].astype(np.float32)
    var = rng.uniform(0.6, 2.0, size=(K, d)).astype(np.float32)
    lw = np.log(rng.dirichlet(np.ones(K))).astype(np.float32)
    return X, mu, var, lw


def _check(ids, resp, R, r, tau, label):
    N, K = R.shape
    order = np.argsort(-R, axis=1, kind="stable")      # ties to the lower index
    Rs = np.take_along_axis(R, order, axis=1)
    worst = 0.0
    for n in range(N):
        kept = ids[n][ids[n] >= 0]
        assert len(set(kept.tolist())) == len(kept), (label, n)
        assert np.all(ids[n][len(kept):] == -1) and np.all(resp[n][len(kept):] == 0), (label, n)
        # values: the GPU responsibility of each kept id
        if len(kept):
            err = np.abs(resp[n][:len(kept)] - R[n, kept])
            worst = max(worst, float(err.max()))
            assert err.max() <= TOL_R, (label, n, err.max())
            assert np.all(np.diff(resp[n][:len(kept)]) <= TOL_R), (label, n)   # descending
            assert np.all(R[n, kept] >= tau - TOL_R), (label, n)
        # the oracle's own selection where it is unambiguous
        want = [order[n, j] for j in range(min(r, K)) if Rs[n, j] >= tau]
        amb = abs(Rs[n, min(r, K) - 1] - Rs[n, min(r, K)]) <= TOL_R if K > r else False
        amb |= bool(np.any(np.abs(Rs[n, :min(r, K) + 1] - tau) <= TOL_R))
        if not amb:
            assert set(kept.tolist()) == set(want), (label, n, kept, want)
        else:
            # still valid: every kept id is within the tolerance of the r best
            floor = Rs[n, min(r, K) - 1] - TOL_R
            assert np.all(R[n, kept] >= min(floor, tau) - TOL_R), (label, n)
    return worst


@pytest.mark.parametrize("N,d,K,dtype,r,tau,flags", [
    (5000, 64, 40, "f32", 3, 0.05, 0),        # tensor cores, one 256-component chunk
    (4100, 128, 300, "bf16", 4, 0.01, 0),     # two chunks, ragged tail of points
    (3000, 32, 600, "f16", 8, 0.0, 0),        # three chunks, pure top-8
    (2500, 128, 256, "f32", 2, 0.2, 0),
    (3000, 16, 12, "f32", 8, 0.0, 0),         # d = 16: CUDA-core kernel, K < r
    (2000, 96, 50, "bf16", 3, 0.05, 0),       # d = 96: CUDA-core kernel
    (5000, 64, 40, "f32", 3, 0.05, 2),        # forced CUDA-core kernel
])
def test_soft_assign_matches_oracle(N, d, K, dtype, r, tau, flags):
    X, mu, var, lw = _case(N + d + K, N, d, K, dtype)
    Xd = torch.from_numpy(X).to(TORCH_DT[dtype]).cuda()
    m, v, l = (torch.from_numpy(a).cuda() for a in (mu, var, lw))
    ws = gmm.Workspace.for_gmm(N, d, K, Xd.dtype)
    ids, resp, ll = gmm.soft_assign(Xd, m, v, l, r, tau, ws, want_loglik=True, flags=flags)
    assert gmm.gmm_last_error(ws) == 0
    ref = oracle.gmm_estep(X, mu, var, lw, want_stats=False, want_R=True)
    assert loglik_err(ll.cpu().numpy(), ref["loglik"]) <= TOL_LOGLIK
    _check(ids.cpu().numpy(), resp.cpu().numpy(), ref["R"], r, tau,
           f"soft-{N}x{d}-K{K}-{dtype}-r{r}")


def test_soft_assign_with_direct_form_components():
    """Collapsed components (scored in the direct form, outside the tensor
    core) take part in the selection: points sitting on a collapsed
    component's mean must list it first."""
    N, d, K = 4000, 128, 100
    X, mu, var, lw = _case(9, N, d, K, "f32", spread=3.0)
    for k, i in [(3, 10), (50, 20), (77, 30)]:
        mu[k] = X[i]
        var[k] = 1e-3
    Xd = torch.from_numpy(X).cuda()
    m, v, l = (torch.from_numpy(a).cuda() for a in (mu, var, lw))
    ws = gmm.Workspace.for_gmm(N, d, K)
    ids, resp, _ = gmm.soft_assign(Xd, m, v, l, 3, 0.0, ws)
    assert gmm.gmm_last_error(ws) == 0
    ids = ids.cpu().numpy()
    for k, i in [(3, 10), (50, 20), (77, 30)]:
        assert ids[i, 0] == k
    ref = oracle.gmm_estep(X, mu, var, lw, want_stats=False, want_R=True)
    _check(ids, resp.cpu().numpy(), ref["R"], 3, 0.0, "soft-direct")
