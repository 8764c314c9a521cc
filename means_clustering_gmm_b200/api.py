"""Python binding of the C ABI, for torch tensors.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libgmm_b200.so.  PyTorch provides the device memory (outputs and
workspaces) and the stream (``torch.cuda.current_stream()`` by default).
"""
from __future__ import annotations

import torch

from . import _lib
from ._lib import (GMM_BF16, GMM_F16, GMM_F32, GMM_FLAG_FORCE_SIMT, GMM_FLAG_FORCE_TWO_SWEEP,
                   GMM_FLAG_NONE, GmmError, check)

_DT = {torch.float32: GMM_F32, torch.bfloat16: GMM_BF16, torch.float16: GMM_F16}

__all__ = ["GMM_FLAG_NONE", "GMM_FLAG_FORCE_TWO_SWEEP", "GMM_FLAG_FORCE_SIMT", "GmmError",
           "Workspace", "gmm_workspace_size", "kmeans_workspace_size", "gmm_em_step",
           "gmm_finalize", "kmeans_step", "gmm_last_error", "em_iteration", "fit"]


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, dtype, shape, name):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_cuda or \
            not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous cuda {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")


def gmm_workspace_size(N: int, d: int, K: int, dtype=torch.float32) -> int:
    return int(_lib.load().gmm_workspace_size(N, d, K, _DT[dtype]))


def kmeans_workspace_size(B: int, N: int, d: int, K: int) -> int:
    return int(_lib.load().kmeans_workspace_size(B, N, d, K))


class Workspace:
    """A device workspace (torch uint8 buffer, 256-byte aligned) with its
    error word cleared once at allocation."""

    def __init__(self, nbytes: int, device=None, stream=None):
        if nbytes <= 0:
            raise ValueError("invalid problem size (workspace size 0)")
        self.nbytes = int(nbytes)
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8,
                               device=device or torch.device("cuda"))
        off = (-self.buf.data_ptr()) % 256
        self.view = self.buf[off:off + self.nbytes]
        check("gmm_workspace_init",
              _lib.load().gmm_workspace_init(self.ptr, self.nbytes, _stream_ptr(stream)))

    @property
    def ptr(self) -> int:
        return self.view.data_ptr()

    @classmethod
    def for_gmm(cls, N, d, K, dtype=torch.float32, device=None):
        return cls(gmm_workspace_size(N, d, K, dtype), device)

    @classmethod
    def for_kmeans(cls, B, N, d, K, device=None):
        return cls(kmeans_workspace_size(B, N, d, K), device)


def gmm_em_step(X: torch.Tensor, means: torch.Tensor, variances: torch.Tensor,
                logw: torch.Tensor, ws: Workspace, stats: torch.Tensor | None = None,
                loglik: torch.Tensor | None = None, loglik_total: torch.Tensor | None = None,
                want_loglik: bool = False, flags: int = GMM_FLAG_NONE, stream=None):
    """Fused E-step + statistics.  Returns (stats [K, 1+2d] fp64 laid out as
    S0|S1|S2 in memory, loglik [N] fp32 or None, loglik_total [1] fp64)."""
    N, d = X.shape
    K = means.shape[0]
    if X.dtype not in _DT or not X.is_cuda or not X.is_contiguous():
        raise ValueError("X must be a contiguous cuda float32/bfloat16/float16 [N, d] tensor")
    _need(means, torch.float32, (K, d), "means")
    _need(variances, torch.float32, (K, d), "vars")
    _need(logw, torch.float32, (K,), "logw")
    dev = X.device
    if stats is None:
        stats = torch.empty(K * (1 + 2 * d), dtype=torch.float64, device=dev)
    if want_loglik and loglik is None:
        loglik = torch.empty(N, dtype=torch.float32, device=dev)
    if loglik_total is None:
        loglik_total = torch.empty(1, dtype=torch.float64, device=dev)
    rc = _lib.load().gmm_em_step(X.data_ptr(), _DT[X.dtype], N, d, K, means.data_ptr(),
                                 variances.data_ptr(), logw.data_ptr(), stats.data_ptr(),
                                 _ptr(loglik), loglik_total.data_ptr(), ws.ptr, ws.nbytes,
                                 int(flags), _stream_ptr(stream))
    check("gmm_em_step", rc)
    return stats, loglik, loglik_total


def gmm_finalize(stats: torch.Tensor, N: int, means: torch.Tensor, variances: torch.Tensor,
                 logw: torch.Tensor, ws: Workspace, var_floor: float = 1e-6, stream=None):
    """M-step finalise; updates means/variances/logw in place."""
    K, d = means.shape
    rc = _lib.load().gmm_finalize(stats.data_ptr(), N, d, K, float(var_floor), means.data_ptr(),
                                  variances.data_ptr(), logw.data_ptr(), ws.ptr, ws.nbytes,
                                  _stream_ptr(stream))
    check("gmm_finalize", rc)
    return means, variances, logw


def gmm_last_error(ws: Workspace, stream=None) -> int:
    """Synchronises the stream; returns and clears the device error word."""
    return int(_lib.load().gmm_last_error(ws.ptr, _stream_ptr(stream)))


def em_iteration(X, means, variances, logw, ws, var_floor=1e-6, want_loglik=False,
                 flags=GMM_FLAG_NONE, stream=None):
    """One EM iteration in place: gmm_em_step then gmm_finalize.  Returns
    (stats, loglik, loglik_total) of the E-step (at the entering params)."""
    out = gmm_em_step(X, means, variances, logw, ws, want_loglik=want_loglik, flags=flags,
                      stream=stream)
    gmm_finalize(out[0], X.shape[0], means, variances, logw, ws, var_floor, stream)
    return out


def fit(X, means, variances, logw, iters: int, ws=None, var_floor=1e-6, flags=GMM_FLAG_NONE,
        stream=None):
    """`iters` EM iterations.  Host tensors are copied to the device first and
    the updated parameters are copied back.  Returns (means, vars, logw,
    loglik_totals [iters] fp64 on the host)."""
    host = not X.is_cuda
    dev = torch.device("cuda")
    Xd = X.to(dev, non_blocking=True) if host else X
    m = means.to(dev, non_blocking=True).clone() if not means.is_cuda else means
    v = variances.to(dev, non_blocking=True).clone() if not variances.is_cuda else variances
    lw = logw.to(dev, non_blocking=True).clone() if not logw.is_cuda else logw
    N, d = Xd.shape
    K = m.shape[0]
    if ws is None:
        ws = Workspace.for_gmm(N, d, K, Xd.dtype)
    totals = torch.empty(iters, dtype=torch.float64, device=dev)
    stats = torch.empty(K * (1 + 2 * d), dtype=torch.float64, device=dev)
    for t in range(iters):
        gmm_em_step(Xd, m, v, lw, ws, stats=stats, loglik_total=totals[t:t + 1], flags=flags,
                    stream=stream)
        gmm_finalize(stats, N, m, v, lw, ws, var_floor, stream)
    if host:
        return m.cpu(), v.cpu(), lw.cpu(), totals.cpu()
    return m, v, lw, totals


def kmeans_step(X: torch.Tensor, centroids: torch.Tensor, ws: Workspace,
                ids: torch.Tensor | None = None, new_centroids: torch.Tensor | None = None,
                counts: torch.Tensor | None = None, inertia: torch.Tensor | None = None,
                flags: int = GMM_FLAG_NONE, stream=None):
    """One Lloyd iteration for B problems: X [B, N, d] (or [N, d]), centroids
    [B, K, d] fp32.  Returns (ids [B, N] int32, new_centroids, counts [B, K]
    int32, inertia [B] fp64)."""
    squeeze = X.dim() == 2
    if squeeze:
        X = X.unsqueeze(0)
        centroids = centroids.unsqueeze(0)
    B, N, d = X.shape
    K = centroids.shape[1]
    if X.dtype not in _DT or not X.is_cuda or not X.is_contiguous():
        raise ValueError("X must be a contiguous cuda float32/bfloat16/float16 tensor")
    _need(centroids, torch.float32, (B, K, d), "centroids")
    dev = X.device
    ids = torch.empty((B, N), dtype=torch.int32, device=dev) if ids is None else ids
    new_centroids = torch.empty_like(centroids) if new_centroids is None else new_centroids
    counts = torch.empty((B, K), dtype=torch.int32, device=dev) if counts is None else counts
    inertia = torch.empty(B, dtype=torch.float64, device=dev) if inertia is None else inertia
    rc = _lib.load().kmeans_step(X.data_ptr(), _DT[X.dtype], B, N, d, K, centroids.data_ptr(),
                                 ids.data_ptr(), new_centroids.data_ptr(), _ptr(counts),
                                 _ptr(inertia), ws.ptr, ws.nbytes, int(flags),
                                 _stream_ptr(stream))
    check("kmeans_step", rc)
    if squeeze:
        return ids[0], new_centroids[0], counts[0], inertia[0]
    return ids, new_centroids, counts, inertia
