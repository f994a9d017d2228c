"""The fp8-layer parity bar is attainable and still discriminating (CPU only).

The float64 layer with fp8 linears, recomputed with bf16 rounding at the points
where the CUDA layer stores bf16 (the four projections, the normalised and
rotated q, k, rho, the attention output, the layer output), must stay well
inside FP8_LAYER_TOL of the fp8 oracle; the layer with unquantised linears
must not.
"""
import numpy as np
import torch

import oracle
from oracle import layer as olayer
from local_linear_attention_streamed_b200 import synth
from _util import FP8_LAYER_TOL, rel_err_fro, small_inputs


def _bf(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64)).float().to(torch.bfloat16).double().numpy()


def _layer_bf16_storage(x, WQ, WK, WV, WR, WO, H):
    B, N, D = x.shape
    d = D // H
    x2 = x.reshape(B * N, D)
    pos = np.arange(N)[None, None, :]

    def heads(y):
        return y.reshape(B, N, H, d).transpose(0, 2, 1, 3)

    def lin(a, W):
        return _bf(olayer.fp8_linear(a, W))

    q = _bf(olayer.rope(olayer.rmsnorm(heads(lin(x2, WQ))), pos))
    k = _bf(olayer.rope(olayer.rmsnorm(heads(lin(x2, WK))), pos))
    v = heads(lin(x2, WV))
    r = _bf(olayer.rope(olayer.rmsnorm(heads(lin(x2, WR))), pos))
    o = _bf(oracle.prefill_ref(q, k, v, r, causal=True))
    return _bf(lin(o.transpose(0, 2, 1, 3).reshape(B * N, D), WO)).reshape(B, N, D)


def test_fp8_layer_bar_is_attainable_and_discriminating():
    B, N, D, H = 2, 160, 256, 2
    _, ref = small_inputs(40 + D + H, synth.layer_specs(B, N, D), synth.BF16, device="cpu")
    args = [ref[n] for n in ("x", "WQ", "WK", "WV", "WR", "WO")]
    want = oracle.layer_fp8_ref(*args, H)
    assert rel_err_fro(_layer_bf16_storage(*args, H), want) <= 0.5 * FP8_LAYER_TOL
    unquantised = oracle.layer_fp8_ref(*args, H, linear=lambda a, W: a @ W)
    assert rel_err_fro(unquantised, want) > 1.5 * FP8_LAYER_TOL
