"""Pure-Python brute force for tiny inputs (N <= ~8, K <= ~4).

TEST INFRASTRUCTURE ONLY.  A second, independent statement of the same
definitions as ``gmm_oracle.c``, written with Python floats, ``math.exp``,
``math.log`` and ``math.fsum`` (correctly rounded sums), so that the C oracle
can be pinned against something other than itself.

Definitions followed (textbook diagonal-covariance GMM; the pages print no
formula, and "Turbo-GMM: FlashAttention-Inspired GPU-Accelerated Gaussian
Mixture Model", abstract, states equivalence to standard EM):
  log N(x; mu, var) = sum_j -1/2 [log(2 pi var_j) + (x_j - mu_j)^2 / var_j]
  s_nk = log w_k + log N(x_n; mu_k, var_k)
  r_nk = exp(s_nk) / sum_k' exp(s_nk')            (direct, no max shift)
  l_n  = log sum_k exp(s_nk)
"""
from __future__ import annotations

import math


def log_density(x, mu, var):
    return math.fsum(-0.5 * (math.log(2.0 * math.pi * v) + (xi - m) ** 2 / v)
                     for xi, m, v in zip(x, mu, var))


def responsibilities(X, means, variances, weights):
    """Returns (R, loglik) for tiny inputs; weights are plain (not log)."""
    R, ll = [], []
    for x in X:
        dens = [w * math.exp(log_density(x, m, v)) for m, v, w in zip(means, variances, weights)]
        tot = math.fsum(dens)
        R.append([p / tot for p in dens])
        ll.append(math.log(tot))
    return R, ll


def em_iteration(X, means, variances, weights):
    """One EM iteration; returns (means, variances, weights, loglik_total)."""
    R, ll = responsibilities(X, means, variances, weights)
    K = len(means)
    d = len(X[0])
    N = len(X)
    new_m, new_v, new_w = [], [], []
    for k in range(K):
        nk = math.fsum(R[n][k] for n in range(N))
        mk = [math.fsum(R[n][k] * X[n][j] for n in range(N)) / nk for j in range(d)]
        vk = [math.fsum(R[n][k] * (X[n][j] - mk[j]) ** 2 for n in range(N)) / nk
              for j in range(d)]
        new_m.append(mk)
        new_v.append(vk)
        new_w.append(nk / N)
    return new_m, new_v, new_w, math.fsum(ll)


def lloyd(X, C):
    """One Lloyd iteration by exhaustive search; ties go to the lowest index."""
    K = len(C)
    d = len(X[0])
    ids = []
    for x in X:
        best, arg = math.inf, -1
        for k in range(K):
            dist = math.fsum((xi - ci) ** 2 for xi, ci in zip(x, C[k]))
            if dist < best:
                best, arg = dist, k
        ids.append(arg)
    newC = []
    for k in range(K):
        members = [X[n] for n in range(len(X)) if ids[n] == k]
        if members:
            newC.append([math.fsum(m[j] for m in members) / len(members) for j in range(d)])
        else:
            newC.append(list(C[k]))
    return ids, newC
