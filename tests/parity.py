"""Comparison helpers for the parity tests (CUDA path vs float64 oracle).

Tolerances (stated for the fused EM step and the Lloyd step):
  * means and variances: relative error <= 1e-5 for fp32 inputs and <= 1e-3 for
    bf16/fp16 inputs, read normwise per tensor: ||gpu - ref||_2 / ||ref||_2;
    and element by element, every (k, j) against the raw second moment the
    sufficient statistics carry it in, m2_kj = mu_kj^2 + var_kj (reference
    values): |d mu_kj| / sqrt(m2_kj) and |d var_kj| / m2_kj, each <= TOL_ELEM
    (the statistics S1 = sum r x and S2 = sum r x^2 are summed with an error
    relative to sum r |x| and sum r x^2, so a mean near zero or a variance far
    below mu^2 has no tighter bound than this; the plain per-element
    |d| / max(|ref|, 1e-6 max|ref|) is reported beside it);
  * per-point log-likelihood: max_n |gpu_n - ref_n| / max(|ref_n|, 1) <= 1e-4;
  * mixture weights: max absolute error <= 1e-5;
  * k-means ids: bit-exact except where the oracle's two smallest squared
    distances differ by less than 1e-3 relative ((d2 - d1) / d1 < 1e-3, d1 > 0);
  * centroids: relative error <= 1e-3, normwise.
"""
from __future__ import annotations

import json
import os

import numpy as np

TOL_PARAM = {"f32": 1e-5, "bf16": 1e-3, "f16": 1e-3}
# Element by element against the raw second moment: 1e-3 for every dtype.
# The kernels compute at ~22-bit precision whatever the input dtype; a single
# component fed by points that sit between two components carries the
# expanded score form's error (about 2^-21 Q_k absolute, Q_k up to 2^12) into
# its responsibilities, so one element can be ~100x the normwise error (the
# largest measured over the GPU suite: 3.2e-4).
TOL_ELEM = {"f32": 1e-3, "bf16": 1e-3, "f16": 1e-3}
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


def plain_elementwise(gpu, ref) -> float:
    """max |gpu - ref| / max(|ref|, 1e-6 max|ref|) over the elements (reported)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    floor = 1e-6 * float(np.max(np.abs(ref)))
    den = np.maximum(np.abs(ref), floor if floor > 0 else 1.0)
    return float(np.max(np.abs(gpu - ref) / den))


def moment_elementwise(gpu_mu, gpu_var, ref_mu, ref_var) -> tuple[float, float]:
    """Per-element errors of the means and variances against the raw second
    moment m2 = mu^2 + var of the reference: (max |d mu| / sqrt(m2),
    max |d var| / m2)."""
    gm = np.asarray(gpu_mu, np.float64)
    gv = np.asarray(gpu_var, np.float64)
    rm = np.asarray(ref_mu, np.float64)
    rv = np.asarray(ref_var, np.float64)
    if rm.size == 0:
        return 0.0, 0.0
    m2 = rm * rm + rv
    return (float(np.max(np.abs(gm - rm) / np.sqrt(m2))),
            float(np.max(np.abs(gv - rv) / m2)))


def _worst_element(gpu, ref) -> dict:
    """Where the largest per-element variance error sits: its component k,
    the component's reference weight and Q_k = sum_j mu_kj^2 / var_kj."""
    rm = np.asarray(ref["means"], np.float64)
    rv = np.asarray(ref["vars"], np.float64)
    if rm.size == 0:
        return {}
    e = np.abs(np.asarray(gpu["vars"], np.float64) - rv) / (rm * rm + rv)
    k, j = np.unravel_index(int(np.argmax(e)), e.shape)
    return {"worst_var_k": int(k), "worst_var_j": int(j),
            "worst_var_w": float(np.exp(np.asarray(ref["logw"], np.float64)[k])),
            "worst_var_Q": float((rm[k] ** 2 / rv[k]).sum())}


def _log(label: str, dtype: str, errs: dict) -> None:
    """Append the measured errors to $GMM_PARITY_LOG (JSON lines), if set."""
    path = os.environ.get("GMM_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"label": label, "dtype": dtype, **errs}) + "\n")


def check_gmm_iteration(gpu: dict, ref: dict, dtype: str, label: str = "") -> dict:
    """gpu/ref dicts with means, vars, logw, loglik.  Asserts the tolerances
    (normwise and element by element) and returns the measured errors."""
    errs = {
        "means": normwise(gpu["means"], ref["means"]),
        "vars": normwise(gpu["vars"], ref["vars"]),
        "weights": weight_err(gpu["logw"], ref["logw"]),
    }
    errs["means_elem"], errs["vars_elem"] = moment_elementwise(
        gpu["means"], gpu["vars"], ref["means"], ref["vars"])
    errs.update(_worst_element(gpu, ref))
    errs["means_plain_elem"] = plain_elementwise(gpu["means"], ref["means"])
    errs["vars_plain_elem"] = plain_elementwise(gpu["vars"], ref["vars"])
    if gpu.get("loglik") is not None:
        errs["loglik"] = loglik_err(gpu["loglik"], ref["loglik"])
    _log(label, dtype, errs)
    tol = TOL_PARAM[dtype]
    assert errs["means"] <= tol, (label, errs)
    assert errs["vars"] <= tol, (label, errs)
    assert errs["means_elem"] <= TOL_ELEM[dtype], (label, errs)
    assert errs["vars_elem"] <= TOL_ELEM[dtype], (label, errs)
    assert errs["weights"] <= TOL_WEIGHT, (label, errs)
    if "loglik" in errs:
        assert errs["loglik"] <= TOL_LOGLIK, (label, errs)
    return errs


def check_stats(gpu: dict, ref: dict, dtype: str, label: str = "") -> dict:
    """Raw statistics S0, S1, S2 against the oracle's, each element against
    the scale it is summed at, with a floor of one point's worth of mass
    (w_k = max(S0_k, 1), m2_kj = S2_kj / S0_k the component's mean square):
      S0: |d S0_k| / w_k
      S1: |d S1_kj| / (w_k sqrt(m2_kj))   (sum r |x| <= sqrt(S0 S2))
      S2: |d S2_kj| / (w_k m2_kj)
    Reported and asserted at TOL_ELEM."""
    r0 = np.asarray(ref["S0"], np.float64)
    r1 = np.asarray(ref["S1"], np.float64)
    r2 = np.asarray(ref["S2"], np.float64)
    g0 = np.asarray(gpu["S0"], np.float64)
    g1 = np.asarray(gpu["S1"], np.float64)
    g2 = np.asarray(gpu["S2"], np.float64)
    tiny = 1e-300
    w = np.maximum(r0, 1.0)
    with np.errstate(divide="ignore", invalid="ignore"):
        m2 = np.where(r0[:, None] > 0, r2 / r0[:, None], 0.0)
    errs = {
        "S0_elem": float(np.max(np.abs(g0 - r0) / w)),
        "S1_elem": float(np.max(np.abs(g1 - r1) / (w[:, None] * np.sqrt(m2) + tiny))),
        "S2_elem": float(np.max(np.abs(g2 - r2) / (w[:, None] * m2 + tiny))),
    }
    e2 = np.abs(g2 - r2) / (w[:, None] * m2 + tiny)
    kk, jj = np.unravel_index(int(np.argmax(e2)), e2.shape)
    errs["worst_S2"] = {"k": int(kk), "j": int(jj), "ref": [float(r0[kk]), float(r1[kk, jj]),
                                                            float(r2[kk, jj])],
                        "gpu": [float(g0[kk]), float(g1[kk, jj]), float(g2[kk, jj])]}
    _log(label + "-stats", dtype, errs)
    errs.pop("worst_S2")
    for k, v in errs.items():
        assert v <= TOL_ELEM[dtype], (label, k, errs)
    return errs
