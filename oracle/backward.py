"""Float64 CPU oracle of the Parallax attention backward pass (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this module.  The CUDA library never calls it, and it never calls
the CUDA library.

The pages train Parallax end to end (rainbus.top 复现评估: pretraining at
0.6B and 1.7B) but print no backward pass; the gradients here are those of
the forward definition itself, taken by float64 automatic differentiation of
a plain, unfused statement of it:

    p_i   = softmax_j(q_i . k_j / sqrt(d))           (causal: j <= i)
    kbar  = sum_j p_ij k_j,   vbar = sum_j p_ij v_j
    out_i = vbar_i - sum_j p_ij ((k_j - kbar_i) . rho_i) (v_j - vbar_i)

(the covariance form of the gist.science summary, "Mecanismo central", with
the boundary factor eta = 0).  The pins in tests/test_oracle.py check these
gradients against central finite differences and against closed forms.
"""
from __future__ import annotations

import numpy as np
import torch


def _hidden_keys(N: int, causal: bool, window=None) -> np.ndarray:
    """[N, N] boolean, True where query i may not see key j: j > i when
    causal, and j <= i - window with a sliding window (which implies causal)."""
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    hidden = (j > i) if (causal or window is not None) else np.zeros((N, N), dtype=bool)
    if window is not None:
        hidden |= j <= i - int(window)
    return hidden


def _forward_torch(Q, K, V, R, causal: bool, window=None):
    """Plain float64 forward over [..., N, d] tensors (all rows at once).

    K and V may have fewer heads than Q (grouped KV heads: query head h reads
    KV head h // (H // Hkv)); they are repeated across each group, so the
    gradients of K and V sum over the group's query heads."""
    if K.dim() == 4 and K.shape[1] != Q.shape[1]:
        G = Q.shape[1] // K.shape[1]
        K = torch.repeat_interleave(K, G, dim=1)
        V = torch.repeat_interleave(V, G, dim=1)
    d = Q.shape[-1]
    N = Q.shape[-2]
    S = Q @ K.transpose(-1, -2) / np.sqrt(d)
    if causal or window is not None:
        S = S.masked_fill(torch.from_numpy(_hidden_keys(N, causal, window)), float("-inf"))
    P = torch.softmax(S, dim=-1)
    kbar = P @ K
    vbar = P @ V
    # probe_ij = (k_j - kbar_i) . rho_i
    probe = R @ K.transpose(-1, -2) - (kbar * R).sum(-1, keepdim=True)
    W = P * probe
    # sum_j p_ij probe_ij (v_j - vbar_i) = (P o probe) V - vbar * sum_j p_ij probe_ij
    corr = W @ V - vbar * W.sum(-1, keepdim=True)
    return vbar - corr


def parallax_forward_ref(Q, K, V, R, causal: bool = True, window=None) -> np.ndarray:
    """Forward output from the same statement (float64), for cross-checks."""
    t = [torch.from_numpy(np.asarray(x, dtype=np.float64)) for x in (Q, K, V, R)]
    with torch.no_grad():
        return _forward_torch(*t, causal, window).numpy()


def prefill_stats_ref(Q, K, V, R, causal: bool = True, window=None):
    """What a training forward saves, per query row (float64), for [B, H, N, d] inputs.

    Returns (vbar [B,H,N,d], lse [B,H,N], tbar [B,H,N]): the softmax mean of the
    visible values, log sum_j exp(q_i . k_j / sqrt(d)) (natural log) and the
    softmax mean of the probe scores t_ij = rho_i . k_j (the weighted means
    that centre the covariance of the gist.science summary's "Mecanismo
    central").
    """
    Q, K, V, R = (np.asarray(x, dtype=np.float64) for x in (Q, K, V, R))
    N, d = Q.shape[-2], Q.shape[-1]
    S = Q @ np.swapaxes(K, -1, -2) / np.sqrt(d)
    if causal or window is not None:
        S = np.where(_hidden_keys(N, causal, window), -np.inf, S)
    smax = S.max(axis=-1, keepdims=True)
    W = np.exp(S - smax)
    omega = W.sum(axis=-1, keepdims=True)
    P = W / omega
    lse = (smax + np.log(omega))[..., 0]
    vbar = P @ V
    tbar = (P * (R @ np.swapaxes(K, -1, -2))).sum(axis=-1)
    return vbar, lse, tbar


def parallax_backward_ref(Q, K, V, R, dO, causal: bool = True, window=None):
    """Gradients (dQ, dK, dV, dR) of sum(out * dO) for inputs [B, H, N, d] (float64);
    ``window`` (None or W >= 1) restricts query i to its last W keys."""
    t = [torch.from_numpy(np.asarray(x, dtype=np.float64)).requires_grad_(True) for x in (Q, K, V, R)]
    out = _forward_torch(*t, causal, window)
    out.backward(torch.from_numpy(np.asarray(dO, dtype=np.float64)))
    return tuple(x.grad.numpy() for x in t)
