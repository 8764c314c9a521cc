"""Comparison helpers for the parity tests (CUDA path vs float64 oracle).

Tolerances (stated for the fused EM step and the Lloyd step):
  * means and variances: relative error <= 1e-5 for fp32 inputs and <= 1e-3 for
    bf16/fp16 inputs, read normwise per tensor: ||gpu - ref||_2 / ||ref||_2;
  * per-point log-likelihood: max_n |gpu_n - ref_n| / max(|ref_n|, 1) <= 1e-4;
  * mixture weights: max absolute error <= 1e-5;
  * k-means ids: bit-exact except where the oracle's two smallest squared
    distances differ by less than 1e-3 relative ((d2 - d1) / d1 < 1e-3, d1 > 0);
  * centroids: relative error <= 1e-3, normwise.
"""
from __future__ import annotations

import numpy as np

TOL_PARAM = {"f32": 1e-5, "bf16": 1e-3, "f16": 1e-3}
TOL_LOGLIK = 1e-4
TOL_WEIGHT = 1e-5
TOL_CENTROID = 1e-3
TIE_GAP = 1e-3


def normwise(gpu, ref) -> float:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref.ravel())
    return float(np.linalg.norm((gpu - ref).ravel()) / (den if den > 0 else 1.0))


def loglik_err(gpu, ref) -> float:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(gpu - ref) / np.maximum(np.abs(ref), 1.0))) if ref.size else 0.0


def weight_err(gpu_logw, ref_logw) -> float:
    return float(np.max(np.abs(np.exp(np.asarray(gpu_logw, np.float64)) -
                               np.exp(np.asarray(ref_logw, np.float64)))))


def near_tie_mask(d1, d2) -> np.ndarray:
    d1 = np.asarray(d1)
    d2 = np.asarray(d2)
    with np.errstate(divide="ignore", invalid="ignore"):
        gap = (d2 - d1) / d1
    return (d1 > 0) & (gap < TIE_GAP)


def check_gmm_iteration(gpu: dict, ref: dict, dtype: str, label: str = "") -> dict:
    """gpu/ref dicts with means, vars, logw, loglik.  Asserts the tolerances
    and returns the measured errors."""
    errs = {
        "means": normwise(gpu["means"], ref["means"]),
        "vars": normwise(gpu["vars"], ref["vars"]),
        "weights": weight_err(gpu["logw"], ref["logw"]),
    }
    if gpu.get("loglik") is not None:
        errs["loglik"] = loglik_err(gpu["loglik"], ref["loglik"])
    tol = TOL_PARAM[dtype]
    assert errs["means"] <= tol, (label, errs)
    assert errs["vars"] <= tol, (label, errs)
    assert errs["weights"] <= TOL_WEIGHT, (label, errs)
    if "loglik" in errs:
        assert errs["loglik"] <= TOL_LOGLIK, (label, errs)
    return errs
