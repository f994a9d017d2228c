"""Float64 CPU oracle for a decode over an fp8 (e4m3) KV cache.

TEST INFRASTRUCTURE ONLY (see ``oracle/parallax.py``).

The pages run the linear layers in dynamic fp8 (rainbus.top summary,
"复现评估": dynamic fp8 for the linears, bf16 for the LM head) and fix no
format for a cached K/V.  The reading here carries "dynamic" over to a cache
that grows one token at a time: every cached key (and value) row of one head
is quantised on its own, when it is written, with its own scale

    s = fp32(max_e |x_e|) / 448                  (448: the largest e4m3 value)
    code_e = e4m3(fp32(x_e) / s)                  (round to nearest, ties to even)

with both divisions in IEEE float32 (the precision the quantiser takes its
rounding decisions in); an all-zero row has s = 0 and zero codes.  The cache
stands for the values code_e * s, and the decode is the plain Parallax decode
(``decode_gqa_ref``) over those values, exactly as the bf16 decode is over the
bf16 values.
"""
from __future__ import annotations

import numpy as np

from .layer import E4M3_MAX, e4m3
from .parallax import decode_gqa_ref


def e4m3_bits(values: np.ndarray) -> np.ndarray:
    """uint8 encodings (sign, 4 exponent bits, 3 mantissa bits) of e4m3 values."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(values, dtype=np.float64)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy().copy()


def e4m3_value(bits: np.ndarray) -> np.ndarray:
    """float64 value of uint8 e4m3 encodings."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def kv_quantize_fp8_ref(X: np.ndarray):
    """Per-row dynamic e4m3 quantisation of cache rows X[..., d].

    Returns (codes uint8 [..., d], scales float32 [...]).
    """
    x32 = np.asarray(X, dtype=np.float64).astype(np.float32)
    amax = np.max(np.abs(x32), axis=-1)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1))
    y = (x32 / safe[..., None]).astype(np.float32)
    y = np.where(s[..., None] > 0, y, np.float32(0))
    return e4m3_bits(e4m3(y.astype(np.float64))), s


def kv_dequantize_fp8_ref(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """The values a quantised cache stands for: code * scale, in float64 (exact)."""
    return e4m3_value(codes) * np.asarray(scales, dtype=np.float64)[..., None]


def decode_fp8kv_ref(q, r, Kcodes, Kscales, Vcodes, Vscales, seqlens, units=None) -> np.ndarray:
    """One decode step over an e4m3 cache: q, r [B, H, d]; codes [B, Hkv, L, d];
    scales [B, Hkv, L]; query head h reads KV head h // (H / Hkv)."""
    K = kv_dequantize_fp8_ref(Kcodes, Kscales)
    V = kv_dequantize_fp8_ref(Vcodes, Vscales)
    return decode_gqa_ref(q, r, K, V, seqlens, units=units)
