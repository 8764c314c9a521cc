"""Runs the CUDA path through the C ABI (via the torch binding) on numpy
inputs and returns numpy outputs, for the parity tests."""
from __future__ import annotations

import numpy as np
import torch

import means_clustering_gmm_b200 as gmm  # noqa: F401  (tests reach it as g.gmm)

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def to_device_x(X32: np.ndarray, dtype: str) -> torch.Tensor:
    """X32 already holds values of `dtype` (rounded once by synth); the cast is exact."""
    return torch.from_numpy(np.ascontiguousarray(X32)).to(TORCH_DT[dtype]).cuda()


def gmm_iteration(Xd: torch.Tensor, means, vars_, logw, flags=0, var_floor=1e-6, ws=None):
    """One E-step + finalise on the GPU.  Returns numpy dict and the error word."""
    N, d = Xd.shape
    K = means.shape[0]
    m = torch.from_numpy(np.ascontiguousarray(means, np.float32)).cuda()
    v = torch.from_numpy(np.ascontiguousarray(vars_, np.float32)).cuda()
    lw = torch.from_numpy(np.ascontiguousarray(logw, np.float32)).cuda()
    if ws is None:
        ws = gmm.Workspace.for_gmm(N, d, K, Xd.dtype)
    stats, ll, tot = gmm.gmm_em_step(Xd, m, v, lw, ws, want_loglik=True, flags=flags)
    gmm.gmm_finalize(stats, N, m, v, lw, ws, var_floor)
    err = gmm.gmm_last_error(ws)
    st = stats.cpu().numpy()
    return {
        "means": m.cpu().numpy(), "vars": v.cpu().numpy(), "logw": lw.cpu().numpy(),
        "loglik": ll.cpu().numpy(), "loglik_total": float(tot.cpu().numpy()[0]),
        "S0": st[:K], "S1": st[K:K + K * d].reshape(K, d), "S2": st[K + K * d:].reshape(K, d),
        "err": err,
    }


def kmeans_iteration(Xd: torch.Tensor, C: np.ndarray, flags=0, ws=None):
    B, N, d = Xd.shape
    K = C.shape[1]
    Ct = torch.from_numpy(np.ascontiguousarray(C, np.float32)).cuda()
    if ws is None:
        ws = gmm.Workspace.for_kmeans(B, N, d, K)
    ids, newC, counts, inertia = gmm.kmeans_step(Xd, Ct, ws, flags=flags)
    err = gmm.gmm_last_error(ws)
    return {"ids": ids.cpu().numpy(), "centroids": newC.cpu().numpy(),
            "counts": counts.cpu().numpy(), "inertia": inertia.cpu().numpy(), "err": err}
