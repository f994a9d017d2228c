"""Float64 CPU oracle for a full Parallax attention layer.

TEST INFRASTRUCTURE ONLY (see ``oracle/parallax.py``).

The layer ("Parallax: Parameterized Local Linear Attention for Language
Modeling"; agihunt.info summary: the model carries an extra R = W_R x beside
Q, K, V, rho gets its own RMSNorm and RoPE on it helps; rainbus.top
reproduction notes: Qwen-3 architecture) is, per token x_t:

    q = x W_Q, k = x W_K, v = x W_V, rho = x W_R      (weights stored [in, out])
    split into H heads of width d
    q, k, rho <- RoPE(RMSNorm(.)) per head             (v untouched)
    o_t = Parallax attention over t' <= t, per head
    y = concat_heads(o) W_O

Readings the pages leave open: RMSNorm over each head's d features with unit
weight and eps = 1e-6 (Qwen-3 style); RoPE in the rotate-half form with
frequencies base^(-2k/d), base 10000, position = token index; RoPE applied
after RMSNorm to q, k and rho alike.  Everything is float64 with no
intermediate rounding.
"""
from __future__ import annotations

import numpy as np

from .parallax import parallax_row

RMS_EPS = 1e-6
ROPE_BASE = 10000.0


def rmsnorm(x: np.ndarray, eps: float = RMS_EPS) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) over the last axis (unit weight)."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def rope(x: np.ndarray, pos: np.ndarray, base: float = ROPE_BASE) -> np.ndarray:
    """Rotate-half RoPE on the last axis; ``pos`` broadcasts against x[..., 0].

    Feature k is paired with feature k + d/2 and the pair is rotated by the
    angle pos * base^(-2k/d).
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    k = np.arange(half, dtype=np.float64)
    inv_freq = base ** (-2.0 * k / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv_freq
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def layer_rows_ref(x, WQ, WK, WV, WR, WO, H: int, rows) -> np.ndarray:
    """Layer output rows y[b, t] for the (b, t) pairs in ``rows``.

    x: float64 [B, N, D]; W*: float64 [D, D] stored [in, out].  Returns
    float64 [len(rows), D].
    """
    x = np.asarray(x, dtype=np.float64)
    B, N, D = x.shape
    d = D // H
    out = []
    cache = {}
    for (b, t) in rows:
        if b not in cache:
            xb = x[b]
            pos = np.arange(N)
            k = xb @ WK
            v = xb @ WV
            kh = k.reshape(N, H, d).transpose(1, 0, 2)
            vh = v.reshape(N, H, d).transpose(1, 0, 2)
            kh = rope(rmsnorm(kh), pos[None, :])
            cache[b] = (kh, vh)
        kh, vh = cache[b]
        xt = x[b, t]
        qh = rope(rmsnorm((xt @ WQ).reshape(H, d)), np.full(H, t))
        rh = rope(rmsnorm((xt @ WR).reshape(H, d)), np.full(H, t))
        o = np.concatenate([parallax_row(qh[h], rh[h], kh[h, :t + 1], vh[h, :t + 1])
                            for h in range(H)])
        out.append(o @ WO)
    return np.stack(out)


def qkr_norm_rope_ref(x, W, H: int) -> np.ndarray:
    """RoPE(RMSNorm(x W)) per head for all tokens: returns [B, H, N, d]."""
    x = np.asarray(x, dtype=np.float64)
    B, N, D = x.shape
    d = D // H
    y = (x @ W).reshape(B, N, H, d).transpose(0, 2, 1, 3)
    return rope(rmsnorm(y), np.arange(N)[None, None, :])
