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
           "gmm_finalize", "kmeans_step", "gmm_last_error", "em_iteration", "fit",
           "fit_workspace_size", "init_kmeans", "init_kmeans_workspace_size",
           "BatchedWorkspace", "gmm_em_step_batched", "gmm_finalize_batched", "soft_assign",
           "point_chunk", "set_point_chunk", "KernelTimer"]


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


def point_chunk(N: int, d: int, K: int, dtype=torch.float32, flags: int = GMM_FLAG_NONE) -> int:
    """Points per chunk of gmm_em_step / soft_assign on this problem (N when
    the call runs in one piece)."""
    n = int(_lib.load().gmm_point_chunk(N, d, K, _DT[dtype], int(flags)))
    if n < 0:
        raise ValueError("invalid problem size")
    return n


def set_point_chunk(points: int) -> None:
    """Cap the points per chunk of later tensor-core calls (0 = automatic)."""
    check("gmm_set_point_chunk", _lib.load().gmm_set_point_chunk(int(points)))


class KernelTimer:
    """Collects the duration of every dominant-kernel region the library
    launches inside the ``with`` block (one per point chunk of a GMM step, one
    per k-means step); ``ms`` holds them in launch order after the block."""

    def __init__(self, cap: int = 1 << 16):
        self.cap = int(cap)
        self.ms: list[float] = []

    def __enter__(self):
        check("gmm_kernel_timer_begin", _lib.load().gmm_kernel_timer_begin())
        return self

    def __exit__(self, *exc):
        import ctypes
        buf = (ctypes.c_double * self.cap)()
        n = ctypes.c_int64(0)
        rc = _lib.load().gmm_kernel_timer_end(buf, self.cap, ctypes.byref(n))
        if exc[0] is None:
            check("gmm_kernel_timer_end", rc)
        self.ms = [float(buf[i]) for i in range(min(int(n.value), self.cap))]
        return False


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


def soft_assign(X: torch.Tensor, means: torch.Tensor, variances: torch.Tensor,
                logw: torch.Tensor, r: int, tau: float, ws: Workspace, want_loglik=False,
                flags: int = GMM_FLAG_NONE, stream=None):
    """Top-r components per point with responsibility >= tau (gmm_soft_assign).
    Returns (ids [N, r] int32 with -1 past the cut, resp [N, r] fp32, loglik
    [N] or None)."""
    N, d = X.shape
    K = means.shape[0]
    if X.dtype not in _DT or not X.is_cuda or not X.is_contiguous():
        raise ValueError("X must be a contiguous cuda float32/bfloat16/float16 [N, d] tensor")
    _need(means, torch.float32, (K, d), "means")
    _need(variances, torch.float32, (K, d), "vars")
    _need(logw, torch.float32, (K,), "logw")
    dev = X.device
    ids = torch.empty((N, r), dtype=torch.int32, device=dev)
    resp = torch.empty((N, r), dtype=torch.float32, device=dev)
    ll = torch.empty(N, dtype=torch.float32, device=dev) if want_loglik else None
    rc = _lib.load().gmm_soft_assign(X.data_ptr(), _DT[X.dtype], N, d, K, means.data_ptr(),
                                     variances.data_ptr(), logw.data_ptr(), int(r), float(tau),
                                     ids.data_ptr(), resp.data_ptr(), _ptr(ll), ws.ptr, ws.nbytes,
                                     int(flags), _stream_ptr(stream))
    check("gmm_soft_assign", rc)
    return ids, resp, ll


class BatchedWorkspace(Workspace):
    """Workspace of gmm_em_step_batched: one EM workspace per problem, every
    problem's error word cleared at allocation."""

    def __init__(self, B: int, N: int, d: int, K: int, dtype=torch.float32, device=None,
                 stream=None):
        lib = _lib.load()
        self.nbytes = int(lib.gmm_batched_workspace_size(B, N, d, K, _DT[dtype]))
        if self.nbytes <= 0:
            raise ValueError("invalid problem size (workspace size 0)")
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8,
                               device=device or torch.device("cuda"))
        off = (-self.buf.data_ptr()) % 256
        self.view = self.buf[off:off + self.nbytes]
        check("gmm_batched_workspace_init",
              lib.gmm_batched_workspace_init(self.ptr, B, N, d, K, _DT[dtype],
                                             _stream_ptr(stream)))


def gmm_em_step_batched(X: torch.Tensor, means: torch.Tensor, variances: torch.Tensor,
                        logw: torch.Tensor, ws: BatchedWorkspace, want_loglik: bool = False,
                        flags: int = GMM_FLAG_NONE, stream=None):
    """Fused E-step + statistics of B independent problems: X [B, N, d],
    means/variances [B, K, d], logw [B, K].  Returns (stats [B, K*(1+2d)]
    fp64, loglik [B, N] or None, loglik_total [B] fp64)."""
    B, N, d = X.shape
    K = means.shape[1]
    if X.dtype not in _DT or not X.is_cuda or not X.is_contiguous():
        raise ValueError("X must be a contiguous cuda float32/bfloat16/float16 [B, N, d] tensor")
    _need(means, torch.float32, (B, K, d), "means")
    _need(variances, torch.float32, (B, K, d), "vars")
    _need(logw, torch.float32, (B, K), "logw")
    dev = X.device
    stats = torch.empty((B, K * (1 + 2 * d)), dtype=torch.float64, device=dev)
    loglik = torch.empty((B, N), dtype=torch.float32, device=dev) if want_loglik else None
    tot = torch.empty(B, dtype=torch.float64, device=dev)
    rc = _lib.load().gmm_em_step_batched(X.data_ptr(), _DT[X.dtype], B, N, d, K,
                                         means.data_ptr(), variances.data_ptr(), logw.data_ptr(),
                                         stats.data_ptr(), _ptr(loglik), tot.data_ptr(), ws.ptr,
                                         ws.nbytes, int(flags), _stream_ptr(stream))
    check("gmm_em_step_batched", rc)
    return stats, loglik, tot


def gmm_finalize_batched(stats: torch.Tensor, N: int, means: torch.Tensor,
                         variances: torch.Tensor, logw: torch.Tensor, ws: Workspace,
                         var_floor: float = 1e-6, stream=None):
    """M-step finalise of B problems in place (one launch)."""
    B, K, d = means.shape
    rc = _lib.load().gmm_finalize_batched(stats.data_ptr(), B, N, d, K, float(var_floor),
                                          means.data_ptr(), variances.data_ptr(), logw.data_ptr(),
                                          ws.ptr, ws.nbytes, _stream_ptr(stream))
    check("gmm_finalize_batched", rc)
    return means, variances, logw


def fit_workspace_size(N: int, d: int, K: int, dtype=torch.float32) -> int:
    return int(_lib.load().gmm_fit_workspace_size(N, d, K, _DT[dtype]))


def fit(X, means, variances, logw, max_iters: int = 100, tol: float = 1e-6, ws=None,
        var_floor=1e-6, flags=GMM_FLAG_NONE, stream=None):
    """EM until |L_t - L_{t-1}| <= tol |L_t| or max_iters iterations, with the
    loop and the test on the device (gmm_fit: one CUDA graph launch).  Host
    tensors are copied to the device first and the fitted parameters are
    copied back.  Returns (means, vars, logw, loglik_trace [iterations run]
    fp64, converged: bool)."""
    host = not X.is_cuda
    dev = torch.device("cuda")
    Xd = X.to(dev, non_blocking=True) if host else X
    if X.dtype not in _DT or not Xd.is_contiguous():
        raise ValueError("X must be a contiguous float32/bfloat16/float16 [N, d] tensor")
    m = means.to(dev, non_blocking=True).clone() if not means.is_cuda else means
    v = variances.to(dev, non_blocking=True).clone() if not variances.is_cuda else variances
    lw = logw.to(dev, non_blocking=True).clone() if not logw.is_cuda else logw
    N, d = Xd.shape
    K = m.shape[0]
    _need(m, torch.float32, (K, d), "means")
    _need(v, torch.float32, (K, d), "vars")
    _need(lw, torch.float32, (K,), "logw")
    if ws is None:
        ws = Workspace(fit_workspace_size(N, d, K, Xd.dtype))
    trace = torch.empty(max_iters, dtype=torch.float64, device=dev)
    info = torch.zeros(2, dtype=torch.int32, device=dev)
    rc = _lib.load().gmm_fit(Xd.data_ptr(), _DT[Xd.dtype], N, d, K, m.data_ptr(), v.data_ptr(),
                             lw.data_ptr(), int(max_iters), float(tol), float(var_floor),
                             trace.data_ptr(), info.data_ptr(), ws.ptr, ws.nbytes, int(flags),
                             _stream_ptr(stream))
    check("gmm_fit", rc)
    code = gmm_last_error(ws, stream)   # synchronises the stream
    if code != 0:
        raise GmmError("gmm_fit (device)", code)
    its, conv = (int(x) for x in info.cpu())
    trace = trace[:its]
    if host:
        return m.cpu(), v.cpu(), lw.cpu(), trace.cpu(), bool(conv)
    return m, v, lw, trace, bool(conv)


def init_kmeans_workspace_size(N: int, d: int, K: int) -> int:
    return int(_lib.load().gmm_init_kmeans_workspace_size(N, d, K))


def init_kmeans(X: torch.Tensor, centroids: torch.Tensor, iters: int = 10, var_floor=1e-6,
                ws=None, want_ids: bool = False, stream=None):
    """GMM start from k-means (gmm_init_kmeans): `iters` Lloyd iterations
    from `centroids` [K, d], then the hard partition's M-step.  Returns
    (means, vars, logw[, ids]) on the device."""
    N, d = X.shape
    K = centroids.shape[0]
    if X.dtype not in _DT or not X.is_cuda or not X.is_contiguous():
        raise ValueError("X must be a contiguous cuda float32/bfloat16/float16 [N, d] tensor")
    _need(centroids, torch.float32, (K, d), "centroids")
    dev = X.device
    m = centroids.clone()
    v = torch.empty_like(m)
    lw = torch.empty(K, dtype=torch.float32, device=dev)
    ids = torch.empty(N, dtype=torch.int32, device=dev) if want_ids else None
    if ws is None:
        ws = Workspace(init_kmeans_workspace_size(N, d, K), device=dev)
    rc = _lib.load().gmm_init_kmeans(X.data_ptr(), _DT[X.dtype], N, d, K, int(iters),
                                     float(var_floor), m.data_ptr(), v.data_ptr(), lw.data_ptr(),
                                     _ptr(ids), ws.ptr, ws.nbytes, _stream_ptr(stream))
    check("gmm_init_kmeans", rc)
    return (m, v, lw, ids) if want_ids else (m, v, lw)


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
