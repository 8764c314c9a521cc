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
