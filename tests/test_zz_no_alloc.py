"""gmm_em_step_static (the EM step whose workspace is the library's static
device scratch, for callers that cannot allocate) against gmm_em_step with a
caller workspace, through the C ABI.  This file sorts last so that it also
runs after every other test in the same process."""
import ctypes

import numpy as np
import pytest
import torch

import means_clustering_gmm_b200 as gmm
from means_clustering_gmm_b200 import _lib
from synth import round_to

GMM_OK, GMM_ERR_UNSUPPORTED = 0, 2
DT = {"f32": 0, "bf16": 1}
TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _case(seed, N, d, K, dtype):
    rng = np.random.default_rng(seed)
    mu_t = rng.normal(0, 3.0, size=(K, d))
    lab = rng.integers(0, K, size=N)
    X = round_to((mu_t[lab] + rng.standard_normal((N, d))).astype(np.float32), dtype)
    mu = X[rng.choice(N, size=K, replace=False)].astype(np.float32)
    var = rng.uniform(0.5, 2.0, size=(K, d)).astype(np.float32)
    lw = np.log(rng.dirichlet(np.ones(K))).astype(np.float32)
    return X, mu, var, lw


def test_rejects_problems_beyond_the_scratch():
    """A workspace above GMM_STATIC_SCRATCH_BYTES is refused before any device
    work (host-side check; the pointers are never dereferenced)."""
    lib = _lib.load()
    N, d, K = 1 << 22, 128, 256
    assert lib.gmm_workspace_size(N, d, K, 0) > (32 << 20)
    fake = ctypes.c_void_p(1 << 20)
    rc = lib.gmm_em_step_static(fake, 0, N, d, K, fake, fake, fake, fake, None, None, None, 0,
                                None)
    assert rc == GMM_ERR_UNSUPPORTED
    assert lib.gmm_em_step_static(fake, 0, 0, d, K, fake, fake, fake, fake, None, None, None, 0,
                                  None) == 1   # GMM_ERR_INVALID_ARG


@pytest.mark.gpu
@pytest.mark.parametrize("shape,dtype", [((4096, 16, 8), "f32"), ((4096, 64, 8), "f32"),
                                         ((5000, 64, 200), "bf16")])
def test_static_scratch_matches_workspace_path(shape, dtype):
    """Two calls in a row on the static scratch reproduce the workspace path's
    statistics and log-likelihoods (both run the same kernels, so the results
    agree far inside the parity tolerances) and report no device error."""
    lib = _lib.load()
    N, d, K = shape
    assert lib.gmm_workspace_size(N, d, K, DT[dtype]) <= (32 << 20)
    X, mu, var, lw = _case(N + d + K, N, d, K, dtype)
    Xd = torch.from_numpy(X).to(TORCH_DT[dtype]).cuda()
    m, v, l = (torch.from_numpy(a).cuda() for a in (mu, var, lw))
    ws = gmm.Workspace.for_gmm(N, d, K, Xd.dtype)
    ref_stats, ref_ll, ref_tot = gmm.gmm_em_step(Xd, m, v, l, ws, want_loglik=True)
    assert gmm.gmm_last_error(ws) == 0
    ref_stats, ref_ll, ref_tot = (t.cpu().numpy() for t in (ref_stats, ref_ll, ref_tot))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        stats = torch.full((K * (1 + 2 * d),), np.nan, dtype=torch.float64, device="cuda")
        ll = torch.full((N,), np.nan, dtype=torch.float32, device="cuda")
        tot = torch.full((1,), np.nan, dtype=torch.float64, device="cuda")
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        rc = lib.gmm_em_step_static(_ptr(Xd), DT[dtype], N, d, K, _ptr(m), _ptr(v), _ptr(l),
                                    _ptr(stats), _ptr(ll), _ptr(tot), _ptr(status), 0, stream)
        assert rc == GMM_OK, _lib.status_string(rc)
        torch.cuda.synchronize()
        assert int(status.item()) == GMM_OK, f"call {call}"
        np.testing.assert_allclose(stats.cpu().numpy(), ref_stats, rtol=1e-12, atol=0,
                                   err_msg=f"call {call}")
        np.testing.assert_allclose(ll.cpu().numpy(), ref_ll, rtol=1e-6, atol=0,
                                   err_msg=f"call {call}")
        np.testing.assert_allclose(tot.cpu().numpy(), ref_tot, rtol=1e-12, err_msg=f"call {call}")
        # a rejected call (misaligned X) returns before it writes to the scratch
        bad = ctypes.c_void_p(Xd.data_ptr() + 4)
        assert lib.gmm_em_step_static(bad, DT[dtype], N, d, K, _ptr(m), _ptr(v), _ptr(l),
                                      _ptr(stats), _ptr(ll), _ptr(tot), _ptr(status), 0,
                                      stream) == 1   # GMM_ERR_INVALID_ARG
