"""Float64 CPU oracle of exact Local Linear Attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this module.

Parallax replaces LLA's per-query solve for the correction vector rho*_i
(which inverts the softmax-weighted key covariance, with a regularisation
lambda whose trade-offs the pages list: gist.science, "Enunciado del
Problema" and "Mecanismo central") by a learned probe.  With the solved probe
the Parallax output is the LLA output; this module states LLA from its own
definition, the local-linear (weighted ridge) regression of the values on the
key-query differences z_j = k_j - q with the softmax weights p_j:

    min_{b, W}  sum_j p_j |v_j - b - W z_j|^2 + lam |W|_F^2,   out = b,

and the probe that the Parallax form needs to reproduce it,

    rho* = (Sigma_KK + lam I)^-1 (kbar - q),   Sigma_KK = sum_j p_j (k_j - kbar)(k_j - kbar)^T.

The pages print neither formula (they name the per-query solve and lambda);
both are the textbook local-linear estimator the test-time-regression
framework they cite refers to.
"""
from __future__ import annotations

import math

import numpy as np


def _softmax_weights(q, K):
    s = (K @ q) / math.sqrt(q.shape[0])
    w = np.exp(s - s.max())
    return w / w.sum()


def lla_row(q, K, V, lam: float) -> np.ndarray:
    """Intercept of the weighted ridge regression of v on [1, k - q] (slope penalised by lam)."""
    q, K, V = (np.asarray(x, dtype=np.float64) for x in (q, K, V))
    n, d = K.shape
    p = _softmax_weights(q, K)
    X = np.hstack([np.ones((n, 1)), K - q[None, :]])
    sw = np.sqrt(p)[:, None]
    A = sw * X
    Y = sw * V
    if lam > 0:
        pen = np.hstack([np.zeros((d, 1)), math.sqrt(lam) * np.eye(d)])
        A = np.vstack([A, pen])
        Y = np.vstack([Y, np.zeros((d, V.shape[1]))])
    beta, *_ = np.linalg.lstsq(A, Y, rcond=None)
    return beta[0]


def lla_probe(q, K, lam: float) -> np.ndarray:
    """rho* = (Sigma_KK + lam I)^-1 (kbar - q) for one query over its visible keys."""
    q, K = np.asarray(q, dtype=np.float64), np.asarray(K, dtype=np.float64)
    p = _softmax_weights(q, K)
    kbar = p @ K
    kc = K - kbar
    S = (kc * p[:, None]).T @ kc
    return np.linalg.solve(S + lam * np.eye(K.shape[1]), kbar - q)


def lla_prefill_ref(Q, K, V, lam: float, causal: bool = True):
    """Exact LLA over [B, H, N, d] inputs: returns (out, R*) with R* the solved probes."""
    B, H, N, d = Q.shape
    out = np.empty(Q.shape[:3] + (V.shape[-1],))
    Rs = np.empty(Q.shape)
    for b in range(B):
        for h in range(H):
            for i in range(N):
                n = i + 1 if causal else N
                out[b, h, i] = lla_row(Q[b, h, i], K[b, h, :n], V[b, h, :n], lam)
                Rs[b, h, i] = lla_probe(Q[b, h, i], K[b, h, :n], lam)
    return out, Rs
