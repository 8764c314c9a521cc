"""The multi-process host logic of a sharded EM fit, on CPU: two gloo ranks,
each holding a contiguous shard of the points, combine their statistics with
the package's all-reduce; the result must equal the statistics of the whole
data set (the oracle's, computed in one process)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from means_clustering_gmm_b200.sharded import allreduce_statistics, shard_bounds


def test_shard_bounds_partition():
    for n in (1, 7, 100, 1001):
        for world in (1, 2, 3, 8):
            spans = [shard_bounds(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [e - s for s, e in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_bounds(10, 2, 2)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, X, mu, var, lw, out_dir):
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        s, e = shard_bounds(X.shape[0], world, rank)
        local = oracle.gmm_estep(X[s:e], mu, var, lw, want_loglik=False)
        stats = torch.from_numpy(local["stats"].copy())
        tot = torch.tensor([local["loglik_total"]], dtype=torch.float64)
        allreduce_statistics(stats, tot)
        np.save(os.path.join(out_dir, f"stats{rank}.npy"), stats.numpy())
        np.save(os.path.join(out_dir, f"tot{rank}.npy"), tot.numpy())
    finally:
        dist.destroy_process_group()


def test_two_rank_statistics_equal_the_whole(tmp_path):
    import oracle
    oracle.build()
    rng = np.random.default_rng(3)
    N, d, K = 1001, 6, 4
    X = rng.normal(size=(N, d)).astype(np.float32)
    mu = X[:K].copy()
    var = np.ones((K, d), np.float32)
    lw = np.full(K, -np.log(K), np.float32)
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), X, mu, var, lw, str(tmp_path)),
                       nprocs=world, start_method="spawn", join=True)
    whole = oracle.gmm_estep(X, mu, var, lw, want_loglik=False)
    for r in range(world):
        stats = np.load(tmp_path / f"stats{r}.npy")
        tot = np.load(tmp_path / f"tot{r}.npy")
        np.testing.assert_allclose(stats, whole["stats"], rtol=1e-12, atol=1e-9)
        assert tot[0] == pytest.approx(whole["loglik_total"], rel=1e-12)
    # both ranks hold bitwise the same totals
    np.testing.assert_array_equal(np.load(tmp_path / "stats0.npy"), np.load(tmp_path / "stats1.npy"))


def _chain_rank(rank, world, port, X, mu, var, lw, iters, out_dir):
    """Each rank: its shard, then `iters` sharded EM iterations through
    sharded.em_iteration, with the oracle's E-step and M-step as the step
    functions (host tensors), the package's all-reduce in between."""
    import oracle
    from means_clustering_gmm_b200 import sharded
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        s, e = shard_bounds(X.shape[0], world, rank)
        Xs = torch.from_numpy(X[s:e])
        m = torch.from_numpy(mu.copy())
        v = torch.from_numpy(var.copy())
        lwt = torch.from_numpy(lw.copy())
        K, d = m.shape
        stats = torch.zeros(K * (1 + 2 * d), dtype=torch.float64)
        tot = torch.zeros(1, dtype=torch.float64)

        def estep(Xr, mm, vv, ll, st, tt):
            r = oracle.gmm_estep(Xr.numpy(), mm.numpy(), vv.numpy(), ll.numpy(),
                                 want_loglik=False)
            st.copy_(torch.from_numpy(r["stats"]))
            tt.fill_(r["loglik_total"])

        def mstep(st, n, mm, vv, ll, vf):
            r = oracle.gmm_mstep(st.numpy(), n, mm.numpy(), vv.numpy(), vf)
            mm.copy_(torch.from_numpy(r["means"]))
            vv.copy_(torch.from_numpy(r["vars"]))
            ll.copy_(torch.from_numpy(r["logw"]))

        totals = []
        for _ in range(iters):
            sharded.em_iteration(Xs, m, v, lwt, None, X.shape[0], stats, tot, estep=estep,
                                 mstep=mstep)
            totals.append(float(tot[0]))
        np.save(os.path.join(out_dir, f"chain{rank}.npy"),
                np.concatenate([m.numpy().ravel(), v.numpy().ravel(), lwt.numpy(), totals]))
    finally:
        dist.destroy_process_group()


def test_two_rank_em_chain_matches_single_process(tmp_path):
    """sharded.em_iteration end to end on two gloo ranks (local E-step, one
    all-reduce, the M-step on every rank), three iterations: both ranks hold
    bitwise the same parameters, equal to three whole-data oracle iterations."""
    import oracle
    oracle.build()
    rng = np.random.default_rng(4)
    N, d, K = 1203, 5, 3
    centres = rng.normal(0, 4, size=(K, d))
    X = centres[rng.integers(0, K, N)] + rng.normal(size=(N, d))
    mu = X[:K].copy()
    var = np.ones((K, d))
    lw = np.full(K, -np.log(K))
    world, iters = 2, 3
    mp.start_processes(_chain_rank, args=(world, _free_port(), X, mu, var, lw, iters,
                                          str(tmp_path)),
                       nprocs=world, start_method="spawn", join=True)
    a, b = (np.load(tmp_path / f"chain{r}.npy") for r in range(world))
    np.testing.assert_array_equal(a, b)
    m, v, l = mu, var, lw
    totals = []
    for _ in range(iters):
        r = oracle.gmm_em_iteration_onepass(X, m, v, l)
        m, v, l = r["means"], r["vars"], r["logw"]
        totals.append(r["loglik_total"])
    whole = np.concatenate([m.ravel(), v.ravel(), l, totals])
    np.testing.assert_allclose(a, whole, rtol=1e-10, atol=1e-12)


def _failing_rank(rank, world, port, out_dir):
    """Rank 1 raises before its collective; rank 0 must get an error from its
    all-reduce (short process-group timeout) instead of waiting for ever."""
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        raise RuntimeError("rank 1 fails before its all-reduce")
    stats = torch.ones(7, dtype=torch.float64)
    try:
        allreduce_statistics(stats)
        outcome = "completed"
    except Exception as exc:   # noqa: BLE001 - any collective error is the signal
        outcome = "error: " + type(exc).__name__
    with open(os.path.join(out_dir, "rank0.txt"), "w") as f:
        f.write(outcome)


def test_failed_rank_is_detected_by_the_others(tmp_path):
    """A rank that dies between steps: the surviving rank's next all-reduce
    ends with an error within the process-group timeout (host-side failure
    detection; no GPU involved)."""
    import multiprocessing
    ctx = multiprocessing.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_failing_rank, args=(r, 2, port, str(tmp_path)))
             for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank did not finish"
    assert procs[1].exitcode != 0
    outcome = (tmp_path / "rank0.txt").read_text()
    assert outcome.startswith("error"), outcome
