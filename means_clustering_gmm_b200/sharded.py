"""Data-parallel EM over point shards: one process per GPU, each holding a
contiguous shard of the points.

The E-step is independent per point and the sufficient statistics are sums
over points ("Turbo-GMM: FlashAttention-Inspired GPU-Accelerated Gaussian
Mixture Model", abstract: responsibilities weight additive sufficient
statistics), so the only exchange per iteration is one all-reduce of the
[K x (1+2d)] fp64 statistics and the scalar total log-likelihood; every rank
then runs the same M-step on the same totals and holds identical parameters.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_bounds(n_total: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous partition of n_total points: rank r gets [start, end), the
    first n_total % world ranks one point more."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    base, extra = divmod(n_total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_statistics(stats: torch.Tensor, loglik_total: torch.Tensor | None = None,
                         group=None) -> None:
    """Sum the per-rank statistics (and the total log-likelihood) over the
    process group, in place.  fp64 throughout; every rank ends with the same
    values."""
    if stats.dtype != torch.float64:
        raise ValueError("statistics must be float64")
    if loglik_total is None:
        dist.all_reduce(stats, op=dist.ReduceOp.SUM, group=group)
        return
    if loglik_total.dtype != torch.float64 or loglik_total.device != stats.device:
        raise ValueError("loglik_total must be float64 on the statistics' device")
    # one collective: statistics and total packed in one buffer
    buf = torch.cat([stats.reshape(-1), loglik_total.reshape(-1)])
    dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)
    stats.reshape(-1).copy_(buf[:stats.numel()])
    loglik_total.reshape(-1).copy_(buf[stats.numel():])


def em_iteration(X_shard: torch.Tensor, means: torch.Tensor, variances: torch.Tensor,
                 logw: torch.Tensor, ws, n_global: int, stats: torch.Tensor,
                 loglik_total: torch.Tensor, var_floor: float = 1e-6, flags: int = 0,
                 group=None, estep=None, mstep=None) -> None:
    """One EM iteration of a sharded fit: the local fused E-step, one
    all-reduce, the M-step on the global totals (parameters updated in place
    on every rank).

    ``estep(X_shard, means, variances, logw, stats, loglik_total)`` and
    ``mstep(stats, n_global, means, variances, logw, var_floor)`` default to
    the library's gmm_em_step and gmm_finalize; the multi-process tests pass
    host implementations to run the same exchange on CPU ranks."""
    from . import api
    if estep is None:
        def estep(X, m, v, lw, st, tot):
            api.gmm_em_step(X, m, v, lw, ws, stats=st, loglik_total=tot, flags=flags)
    if mstep is None:
        def mstep(st, n, m, v, lw, vf):
            api.gmm_finalize(st, n, m, v, lw, ws, vf)
    estep(X_shard, means, variances, logw, stats, loglik_total)
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        allreduce_statistics(stats, loglik_total, group)
    mstep(stats, n_global, means, variances, logw, var_floor)
