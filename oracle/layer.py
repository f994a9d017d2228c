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


# ---------------------------------------------------------------------------
# fp8 linear layers.  The pages' pretraining runs the linear layers in dynamic
# fp8 (rainbus.top, 复现评估: dynamic fp8 for the linear layers, bf16 for the
# LM head).  Reading: "dynamic" = one scale per tensor per call, s = max|a| /
# 448 (the largest e4m3 value), every operand of a linear (the activation and
# the weight) rounded to e4m3 (round to nearest, ties to even) after division
# by its scale, products accumulated exactly, the sum scaled back by s_a s_w.
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3(a: np.ndarray) -> np.ndarray:
    """Round to the nearest float8 e4m3 value (ties to even); |a| <= 448 expected."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    return t.to(torch.float8_e4m3fn).to(torch.float64).numpy()


def fp8_per_tensor(a: np.ndarray):
    """Dynamic per-tensor e4m3 quantisation: returns (e4m3 codes as float64, scale)."""
    a = np.asarray(a, dtype=np.float64)
    amax = float(np.max(np.abs(a)))
    s = amax / E4M3_MAX if amax > 0 else 1.0
    return e4m3(a / s), s


def fp8_linear(a: np.ndarray, W: np.ndarray) -> np.ndarray:
    """a @ W with both operands quantised per tensor to e4m3 (exact accumulation)."""
    qa, sa = fp8_per_tensor(a)
    qw, sw = fp8_per_tensor(W)
    return (qa @ qw) * (sa * sw)


def layer_fp8_ref(x, WQ, WK, WV, WR, WO, H: int, linear=fp8_linear) -> np.ndarray:
    """The whole layer output [B, N, D] with fp8 linears (float64 elsewhere).

    The scale of the attention output (the input of W_O) depends on every
    token of the batch, so this oracle computes all rows.
    """
    x = np.asarray(x, dtype=np.float64)
    B, N, D = x.shape
    d = D // H
    x2 = x.reshape(B * N, D)
    pos = np.arange(N)[None, None, :]

    def heads(y):
        return y.reshape(B, N, H, d).transpose(0, 2, 1, 3)

    q = rope(rmsnorm(heads(linear(x2, WQ))), pos)
    k = rope(rmsnorm(heads(linear(x2, WK))), pos)
    v = heads(linear(x2, WV))
    r = rope(rmsnorm(heads(linear(x2, WR))), pos)
    o = np.empty((B, H, N, d))
    for b in range(B):
        for h in range(H):
            for t in range(N):
                o[b, h, t] = parallax_row(q[b, h, t], r[b, h, t], k[b, h, :t + 1], v[b, h, :t + 1])
    merged = o.transpose(0, 2, 1, 3).reshape(B * N, D)
    return linear(merged, WO).reshape(B, N, D)
