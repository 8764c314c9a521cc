"""Batched GMM (gmm_em_step_batched / gmm_finalize_batched): B independent
mixtures through the same fused kernels.  Every problem must equal a
separate gmm_em_step call bit for bit and match the oracle."""
import numpy as np
import pytest
import torch

import means_clustering_gmm_b200 as gmm
import oracle
from synth import round_to

from .parity import check_gmm_iteration

pytestmark = pytest.mark.gpu
TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def _problems(seed, B, N, d, K, dtype):
    rng = np.random.default_rng(seed)
    X = np.empty((B, N, d), np.float32)
    mu = np.empty((B, K, d), np.float32)
    var = np.empty((B, K, d), np.float32)
    lw = np.empty((B, K), np.float32)
    for b in range(B):
        centres = rng.normal(0, 2.5, size=(K, d))
        X[b] = centres[rng.integers(0, K, N)] + rng.uniform(0.4, 1.2) * rng.standard_normal((N, d))
        mu[b] = X[b, rng.choice(N, K, replace=False)]
        var[b] = rng.uniform(0.5, 2.0, size=(K, d))
        lw[b] = np.log(rng.dirichlet(np.ones(K)))
    return round_to(X, dtype), mu, var, lw


@pytest.mark.parametrize("B,N,d,K,dtype", [(4, 5000, 64, 40, "f32"), (3, 3001, 128, 200, "bf16"),
                                           (2, 4100, 32, 300, "f16"), (5, 777, 16, 7, "f32"),
                                           (8, 8192, 128, 256, "f16")])
def test_batched_equals_separate_calls_and_oracle(B, N, d, K, dtype):
    X, mu, var, lw = _problems(B * 1000 + K, B, N, d, K, dtype)
    Xd = torch.from_numpy(X).to(TORCH_DT[dtype]).cuda()
    m, v, l = (torch.from_numpy(a).cuda() for a in (mu, var, lw))
    ws = gmm.BatchedWorkspace(B, N, d, K, Xd.dtype)
    stats, ll, tot = gmm.gmm_em_step_batched(Xd, m, v, l, ws, want_loglik=True)
    stats_c, ll_c, tot_c = stats.clone(), ll.clone(), tot.clone()
    gmm.gmm_finalize_batched(stats, N, m, v, l, ws)
    assert gmm.gmm_last_error(ws) == 0
    for b in range(B):
        # the same problem as a separate call: bitwise equal
        wsb = gmm.Workspace.for_gmm(N, d, K, Xd.dtype)
        mb, vb, lb = (torch.from_numpy(a[b]).cuda() for a in (mu, var, lw))
        sb, llb, tb = gmm.gmm_em_step(Xd[b], mb, vb, lb, wsb, want_loglik=True)
        gmm.gmm_finalize(sb, N, mb, vb, lb, wsb)
        assert gmm.gmm_last_error(wsb) == 0
        assert torch.equal(sb, stats_c[b]) and torch.equal(llb, ll_c[b])
        assert torch.equal(tb[0], tot_c[b])
        assert torch.equal(mb, m[b]) and torch.equal(vb, v[b]) and torch.equal(lb, l[b])
        ref = oracle.gmm_em_iteration(X[b], mu[b], var[b], lw[b])
        got = {"means": m[b].cpu().numpy(), "vars": v[b].cpu().numpy(),
               "logw": l[b].cpu().numpy(), "loglik": ll_c[b].cpu().numpy()}
        check_gmm_iteration(got, ref, dtype, f"batched-{B}x{N}x{d}-K{K}-{dtype}-p{b}")


def test_batched_error_of_one_problem_is_reported():
    """A NaN variance in problem 2 of 4 is reported once for the batch; the
    next batched call on the same workspace reports nothing."""
    B, N, d, K = 4, 2000, 64, 10
    X, mu, var, lw = _problems(5, B, N, d, K, "f32")
    Xd = torch.from_numpy(X).cuda()
    bad = var.copy()
    bad[2, 1, 3] = np.nan
    ws = gmm.BatchedWorkspace(B, N, d, K)
    m, l = torch.from_numpy(mu).cuda(), torch.from_numpy(lw).cuda()
    gmm.gmm_em_step_batched(Xd, m, torch.from_numpy(bad).cuda(), l, ws)
    assert gmm.gmm_last_error(ws) == 5   # GMM_ERR_NONFINITE
    gmm.gmm_em_step_batched(Xd, m, torch.from_numpy(var).cuda(), l, ws)
    assert gmm.gmm_last_error(ws) == 0
