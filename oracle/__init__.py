"""Float64 CPU oracle for the fused GMM-EM / Lloyd k-means hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product library
(``means_clustering_gmm_b200``) never imports it and shares no code with it.

``gmm_oracle.c`` holds the arithmetic (plain C, float64, OpenMP over fixed row
blocks).  This module compiles it with gcc on first use and wraps it with
numpy.  ``brute`` is a second, independent pure-Python implementation for tiny
inputs, used to pin the C oracle.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gmm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile gmm_oracle.c into liboracle.so next to it (gcc, -fopenmp)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            dp = ctypes.POINTER(ctypes.c_double)
            i64 = ctypes.c_int64
            lib.oracle_num_threads.restype = ctypes.c_int
            lib.oracle_gmm_estep.argtypes = [dp, i64, ctypes.c_int, ctypes.c_int, dp, dp, dp,
                                             dp, dp, dp, dp]
            lib.oracle_gmm_estep.restype = ctypes.c_int
            lib.oracle_gmm_em_iteration.argtypes = [dp, i64, ctypes.c_int, ctypes.c_int, dp, dp,
                                                    dp, ctypes.c_double, dp, dp, dp, dp, dp, dp]
            lib.oracle_gmm_em_iteration.restype = ctypes.c_int
            lib.oracle_gmm_mstep.argtypes = [dp, i64, ctypes.c_int, ctypes.c_int, dp, dp,
                                             ctypes.c_double, dp, dp, dp]
            lib.oracle_gmm_mstep.restype = ctypes.c_int
            lib.oracle_gmm_hard_mstep.argtypes = [dp, i64, ctypes.c_int, ctypes.c_int,
                                                  ctypes.POINTER(ctypes.c_int32), dp,
                                                  ctypes.c_double, dp, dp, dp]
            lib.oracle_gmm_hard_mstep.restype = ctypes.c_int
            lib.oracle_kmeans_step.argtypes = [dp, ctypes.c_int, i64, ctypes.c_int, ctypes.c_int,
                                               dp, ctypes.POINTER(ctypes.c_int32), dp, dp, dp,
                                               ctypes.POINTER(ctypes.c_int64), dp]
            lib.oracle_kmeans_step.restype = ctypes.c_int
            lib.oracle_kmeans_update.argtypes = [dp, ctypes.c_int, i64, ctypes.c_int,
                                                 ctypes.c_int, ctypes.POINTER(ctypes.c_int32),
                                                 dp, dp, ctypes.POINTER(ctypes.c_int64)]
            lib.oracle_kmeans_update.restype = ctypes.c_int
            _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def gmm_estep(X, means, variances, logw, want_stats=True, want_loglik=True, want_R=False):
    """E-step at the given parameters.

    Returns a dict with ``stats`` (K x (1+2d): S0 | S1 | S2, raw moments),
    ``loglik`` [N], ``loglik_total`` and optionally ``R`` [N x K].
    """
    X = _f64(X)
    N, d = X.shape
    mu = _f64(means)
    var = _f64(variances)
    lw = _f64(logw)
    K = mu.shape[0]
    assert mu.shape == (K, d) and var.shape == (K, d) and lw.shape == (K,)
    stats = np.zeros(K * (1 + 2 * d)) if want_stats else None
    ll = np.zeros(N) if want_loglik else None
    tot = np.zeros(1)
    R = np.zeros((N, K)) if want_R else None
    rc = _load().oracle_gmm_estep(_p(X), N, d, K, _p(mu), _p(var), _p(lw), _p(stats), _p(ll),
                                  _p(tot), _p(R))
    if rc:
        raise RuntimeError(f"oracle_gmm_estep failed ({rc})")
    out = {"loglik_total": float(tot[0])}
    if want_stats:
        out["stats"] = stats.reshape(-1)
        out["S0"] = stats[:K]
        out["S1"] = stats[K:K + K * d].reshape(K, d)
        out["S2"] = stats[K + K * d:].reshape(K, d)
    if want_loglik:
        out["loglik"] = ll
    if want_R:
        out["R"] = R
    return out


def gmm_em_iteration(X, means, variances, logw, var_floor=1e-6):
    """One EM iteration (E-step then M-step with two-pass variances)."""
    X = _f64(X)
    N, d = X.shape
    mu = _f64(means)
    var = _f64(variances)
    lw = _f64(logw)
    K = mu.shape[0]
    mu_o = np.zeros((K, d))
    var_o = np.zeros((K, d))
    lw_o = np.zeros(K)
    nk = np.zeros(K)
    ll = np.zeros(N)
    tot = np.zeros(1)
    rc = _load().oracle_gmm_em_iteration(_p(X), N, d, K, _p(mu), _p(var), _p(lw),
                                         float(var_floor), _p(mu_o), _p(var_o), _p(lw_o),
                                         _p(nk), _p(ll), _p(tot))
    if rc:
        raise RuntimeError(f"oracle_gmm_em_iteration failed ({rc})")
    return {"means": mu_o, "vars": var_o, "logw": lw_o, "Nk": nk, "loglik": ll,
            "loglik_total": float(tot[0])}


def gmm_mstep(stats, N, means, variances, var_floor=1e-6):
    """M-step from raw statistics (S0 | S1 | S2, as gmm_estep returns them),
    one-pass variance in float64.  Returns means, vars, logw."""
    mu = _f64(means)
    var = _f64(variances)
    K, d = mu.shape
    st = _f64(stats).reshape(-1)
    assert st.size == K * (1 + 2 * d)
    mu_o = np.zeros((K, d))
    var_o = np.zeros((K, d))
    lw_o = np.zeros(K)
    rc = _load().oracle_gmm_mstep(_p(st), int(N), d, K, _p(mu), _p(var), float(var_floor),
                                  _p(mu_o), _p(var_o), _p(lw_o))
    if rc:
        raise RuntimeError(f"oracle_gmm_mstep failed ({rc})")
    return {"means": mu_o, "vars": var_o, "logw": lw_o}


def gmm_em_iteration_onepass(X, means, variances, logw, var_floor=1e-6):
    """One EM iteration that scores the points once: gmm_estep, then the
    one-pass M-step from its statistics.  Also returns the statistics."""
    e = gmm_estep(X, means, variances, logw)
    m = gmm_mstep(e["stats"], np.asarray(X).shape[0], means, variances, var_floor)
    return {**m, "loglik": e["loglik"], "loglik_total": e["loglik_total"], "S0": e["S0"],
            "S1": e["S1"], "S2": e["S2"]}


def gmm_hard_mstep(X, ids, C, var_floor=1e-6):
    """GMM parameters of a hard partition (X [N, d], ids [N], fallback
    centroids C [K, d]): member means, member variances, weights
    max(n_k, 1) / (N + empty).  Returns means, vars, logw."""
    X = _f64(X)
    C = _f64(C)
    N, d = X.shape
    K = C.shape[0]
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    mu_o = np.zeros((K, d))
    var_o = np.zeros((K, d))
    lw_o = np.zeros(K)
    rc = _load().oracle_gmm_hard_mstep(_p(X), N, d, K,
                                       ids.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                       _p(C), float(var_floor), _p(mu_o), _p(var_o), _p(lw_o))
    if rc:
        raise RuntimeError(f"oracle_gmm_hard_mstep failed ({rc})")
    return {"means": mu_o, "vars": var_o, "logw": lw_o}


def kmeans_step(X, C):
    """One Lloyd iteration for B independent problems.

    X: [B, N, d], C: [B, K, d].  Returns ids [B, N] (int32), d1/d2 (smallest and
    second-smallest squared distances), centroids [B, K, d], counts [B, K],
    inertia [B].
    """
    X = _f64(X)
    C = _f64(C)
    if X.ndim == 2:
        X = X[None]
        C = C[None]
    B, N, d = X.shape
    K = C.shape[1]
    ids = np.zeros((B, N), dtype=np.int32)
    d1 = np.zeros((B, N))
    d2 = np.zeros((B, N))
    Co = np.zeros((B, K, d))
    cnt = np.zeros((B, K), dtype=np.int64)
    inert = np.zeros(B)
    rc = _load().oracle_kmeans_step(_p(X), B, N, d, K, _p(C),
                                    ids.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                    _p(d1), _p(d2), _p(Co),
                                    cnt.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                    _p(inert))
    if rc:
        raise RuntimeError(f"oracle_kmeans_step failed ({rc})")
    return {"ids": ids, "d1": d1, "d2": d2, "centroids": Co, "counts": cnt, "inertia": inert}


def kmeans_update(X, ids, C):
    """Centroid update for given ids (X [B, N, d], ids [B, N], C [B, K, d]):
    mean of the members, empty clusters keep C.  Returns (centroids, counts)."""
    X = _f64(X)
    C = _f64(C)
    if X.ndim == 2:
        X, C = X[None], C[None]
        ids = np.asarray(ids)[None]
    B, N, d = X.shape
    K = C.shape[1]
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    Co = np.zeros((B, K, d))
    cnt = np.zeros((B, K), dtype=np.int64)
    rc = _load().oracle_kmeans_update(_p(X), B, N, d, K,
                                      ids.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                      _p(C), _p(Co),
                                      cnt.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)))
    if rc:
        raise RuntimeError(f"oracle_kmeans_update failed ({rc})")
    return Co, cnt
