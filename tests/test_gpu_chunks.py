"""Point chunks of the tensor-core path: a step over N points runs as
consecutive chunks of rows, each with its own direct-form score block, X
scale and partial statistics, added in chunk order (gmm_point_chunk,
gmm_set_point_chunk).  Parity with the float64 oracle under chunk sizes
that leave a ragged last chunk, in every tensor-core regime, with
ill-conditioned (direct-form) components whose points sit in different
chunks; the chunked and one-piece runs agree to the fp32 accumulation order
of the statistics."""
import numpy as np
import pytest
import torch

import means_clustering_gmm_b200 as gmm
import oracle
from synth import round_to

from .parity import TOL_LOGLIK, check_gmm_iteration, loglik_err, normwise

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    from . import gpu_helpers
    return gpu_helpers


@pytest.fixture
def chunked():
    """Sets the chunk cap for one test and restores the automatic size."""
    yield gmm.set_point_chunk
    gmm.set_point_chunk(0)


def _case(seed, N, d, K, dtype, spread=3.0):
    rng = np.random.default_rng(seed)
    mu_t = rng.normal(0, spread, size=(K, d))
    lab = rng.integers(0, K, size=N)
    X = (mu_t[lab] + rng.uniform(0.4, 1.2, size=(K, d))[lab] *
         rng.standard_normal((N, d))).astype(np.float32)
    X = round_to(X, dtype)
    mu = X[rng.choice(N, size=K, replace=False)].astype(np.float32)
    var = rng.uniform(0.5, 2.0, size=(K, d)).astype(np.float32)
    lw = np.log(rng.dirichlet(np.ones(K))).astype(np.float32)
    # collapsed components on points of the first, a middle and the last chunk
    for k, i in [(1, 17), (K // 2, N // 2 + 3), (K - 2, N - 5)]:
        mu[k] = X[i]
        var[k] = 1e-5
    return X, mu, var, lw


# (N, d, K, dtype, chunk cap): the cap is rounded up to a multiple of 128
CASES = [
    (40000, 128, 256, "f32", 12000),   # two-CTA cluster kernel, 4 chunks (last 3,904 points)
    (30000, 64, 100, "f32", 10000),    # one-CTA kernel, 3 chunks + 384 points
    (9000, 128, 300, "bf16", 2500),    # two sweeps, 4 chunks
    (20000, 64, 2048, "f32", 6000),    # two sweeps over 2048 components
    (50001, 32, 16, "bf16", 15000),    # small-mixture kernel, ragged last chunk
    (12000, 32, 24, "f16", 4000),      # small-mixture kernel, 24 components
]


@pytest.mark.parametrize("N,d,K,dtype,cap", CASES)
def test_chunked_step_matches_oracle(g, chunked, N, d, K, dtype, cap):
    X, mu, var, lw = _case(N + 3 * K + d, N, d, K, dtype)
    Xd = g.to_device_x(X, dtype)
    whole = g.gmm_iteration(Xd, mu, var, lw)
    chunked(cap)
    c = gmm.point_chunk(N, d, K, Xd.dtype)
    assert c == -(-cap // 128) * 128 and c < N
    out = g.gmm_iteration(Xd, mu, var, lw)
    assert out["err"] == 0 and whole["err"] == 0
    ref = oracle.gmm_em_iteration(X, mu, var, lw)
    label = f"chunked-{N}x{d}-K{K}-{dtype}-c{c}"
    check_gmm_iteration(out, ref, dtype, label)
    assert out["loglik_total"] == pytest.approx(ref["loglik_total"], rel=1e-6)
    # against the one-piece run: the per-point work is the same up to the X
    # scale of each chunk; the statistics differ by their accumulation order
    assert loglik_err(out["loglik"], whole["loglik"]) <= TOL_LOGLIK / 10
    for k in ("S0", "S1", "S2"):
        assert normwise(out[k], whole[k]) <= 1e-5, (label, k)
    assert out["loglik_total"] == pytest.approx(whole["loglik_total"], rel=1e-6)


@pytest.mark.parametrize("N,d,K,dtype", [(257, 128, 256, "f32"), (257, 64, 100, "f32"),
                                         (385, 128, 300, "bf16"), (257, 32, 16, "bf16")])
def test_one_point_last_chunk(g, chunked, N, d, K, dtype):
    """Chunks of 128 points over N = 2 or 3 chunks + 1 (N >= K, the means are
    drawn from the points): the last chunk holds one point (one partial tile
    through every kernel of the sequence)."""
    X, mu, var, lw = _case(600 + K, N, d, K, dtype)
    chunked(128)
    assert gmm.point_chunk(N, d, K, g.TORCH_DT[dtype]) == 128
    out = g.gmm_iteration(g.to_device_x(X, dtype), mu, var, lw)
    assert out["err"] == 0
    ref = oracle.gmm_em_iteration(X, mu, var, lw)
    check_gmm_iteration(out, ref, dtype, f"one-point-last-chunk-d{d}-K{K}-{dtype}")
    assert out["loglik_total"] == pytest.approx(ref["loglik_total"], rel=1e-6)


def test_chunked_step_is_deterministic(g, chunked):
    X, mu, var, lw = _case(7, 30000, 128, 256, "f32")
    Xd = g.to_device_x(X, "f32")
    chunked(7000)
    a = g.gmm_iteration(Xd, mu, var, lw)
    b = g.gmm_iteration(Xd, mu, var, lw)
    assert a["err"] == 0
    for k in ["means", "vars", "logw", "loglik", "S0", "S1", "S2"]:
        np.testing.assert_array_equal(a[k], b[k])
    assert a["loglik_total"] == b["loglik_total"]


def test_collecting_timer_sees_one_region_per_chunk(g, chunked):
    N, d, K = 30000, 128, 256
    X, mu, var, lw = _case(8, N, d, K, "f32")
    Xd = g.to_device_x(X, "f32")
    chunked(8000)
    n_chunks = -(-N // gmm.point_chunk(N, d, K))
    assert n_chunks == 4
    with gmm.KernelTimer() as t:
        g.gmm_iteration(Xd, mu, var, lw)
        torch.cuda.synchronize()
    assert len(t.ms) == n_chunks
    assert all(ms > 0 for ms in t.ms)
    gmm.set_point_chunk(0)
    with gmm.KernelTimer() as t:
        g.gmm_iteration(Xd, mu, var, lw)
    assert len(t.ms) == 1


def test_chunked_soft_assign_matches_one_piece(g, chunked):
    """gmm_soft_assign runs chunk by chunk as well; its selection and l_n
    match the one-piece run (same per-point work up to the chunk's X scale)
    and the oracle's log-likelihood."""
    N, d, K, r = 9000, 128, 300, 4
    X, mu, var, lw = _case(9, N, d, K, "f32")
    Xd = g.to_device_x(X, "f32")
    m, v, l = (torch.from_numpy(a).cuda() for a in (mu, var, lw))
    ws = gmm.Workspace.for_gmm(N, d, K)
    ids0, resp0, ll0 = gmm.soft_assign(Xd, m, v, l, r, 0.01, ws, want_loglik=True)
    chunked(2000)
    ids1, resp1, ll1 = gmm.soft_assign(Xd, m, v, l, r, 0.01, ws, want_loglik=True)
    assert gmm.gmm_last_error(ws) == 0
    ref = oracle.gmm_estep(X, mu, var, lw, want_stats=False, want_R=False)
    assert loglik_err(ll1.cpu().numpy(), ref["loglik"]) <= TOL_LOGLIK
    assert loglik_err(ll1.cpu().numpy(), ll0.cpu().numpy()) <= TOL_LOGLIK / 10
    r0, r1 = resp0.cpu().numpy(), resp1.cpu().numpy()
    assert np.abs(r0 - r1).max() <= 1e-4
    i0, i1 = ids0.cpu().numpy(), ids1.cpu().numpy()
    # ids agree wherever the responsibilities are not within the tolerance of a tie
    gaps = np.abs(np.diff(r0, axis=1)).min(axis=1)
    clear = gaps > 1e-4
    np.testing.assert_array_equal(i0[clear], i1[clear])


def test_chunked_fit_equals_chunked_host_loop(g, chunked):
    """gmm_fit captures the chunked step into its graph: the device loop and
    a host loop of the same length agree bit for bit, L never decreases, and
    the end point is an EM fixed point per the oracle."""
    N, d, K = 30000, 128, 256
    X, mu, var, lw = _case(41, N, d, K, "f32")
    chunked(7000)
    Xd = g.to_device_x(X, "f32")
    m0, v0, l0 = (torch.from_numpy(a).cuda() for a in (mu, var, lw))
    m, v, l, trace, conv = gmm.fit(Xd, m0, v0, l0, max_iters=8, tol=1e-7)
    tr = trace.cpu().numpy()
    assert 2 <= len(tr) <= 8
    assert np.all(np.diff(tr) >= -1e-6 * np.abs(tr[1:])), np.diff(tr).min()
    hm, hv, hl = (torch.from_numpy(a).cuda() for a in (mu, var, lw))
    ws = gmm.Workspace.for_gmm(N, d, K)
    for _ in range(len(tr)):
        gmm.em_iteration(Xd, hm, hv, hl, ws)
    assert gmm.gmm_last_error(ws) == 0
    assert torch.equal(m, hm) and torch.equal(v, hv) and torch.equal(l, hl)
    nxt = g.gmm_iteration(Xd, m.cpu().numpy(), v.cpu().numpy(), l.cpu().numpy())
    assert nxt["err"] == 0
    ref = oracle.gmm_em_iteration(X, m.cpu().numpy(), v.cpu().numpy(), l.cpu().numpy())
    check_gmm_iteration(nxt, ref, "f32", "chunked-fit-last")


def test_chunked_batched_equals_separate_calls(g, chunked):
    """Every problem of a batch runs in chunks like a separate call; the
    batch equals the separate calls bit for bit and matches the oracle."""
    B, N, d, K = 2, 20000, 64, 100
    chunked(6000)
    Xs, mus, vs, lws = [], [], [], []
    for b in range(B):
        X, mu, var, lw = _case(50 + b, N, d, K, "bf16")
        Xs.append(X); mus.append(mu); vs.append(var); lws.append(lw)
    X, mu, var, lw = (np.stack(a) for a in (Xs, mus, vs, lws))
    Xd = torch.from_numpy(X).to(torch.bfloat16).cuda()
    m, v, l = (torch.from_numpy(a).cuda() for a in (mu, var, lw))
    ws = gmm.BatchedWorkspace(B, N, d, K, Xd.dtype)
    stats, ll, tot = gmm.gmm_em_step_batched(Xd, m, v, l, ws, want_loglik=True)
    assert gmm.gmm_last_error(ws) == 0
    for b in range(B):
        wsb = gmm.Workspace.for_gmm(N, d, K, Xd.dtype)
        mb, vb, lb = (torch.from_numpy(a[b]).cuda() for a in (mu, var, lw))
        sb, llb, tb = gmm.gmm_em_step(Xd[b], mb, vb, lb, wsb, want_loglik=True)
        assert gmm.gmm_last_error(wsb) == 0
        assert torch.equal(sb, stats[b]) and torch.equal(llb, ll[b]) and torch.equal(tb[0], tot[b])
        ref = oracle.gmm_estep(X[b], mu[b], var[b], lw[b])
        assert loglik_err(ll[b].cpu().numpy(), ref["loglik"]) <= TOL_LOGLIK
        assert normwise(stats[b].cpu().numpy(), ref["stats"].ravel()) <= 1e-3
