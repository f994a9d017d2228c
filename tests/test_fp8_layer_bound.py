"""The fp8-layer parity bars are attainable and still discriminating (CPU only).

The float64 layer with fp8 linears, recomputed with bf16 rounding at the points
where the CUDA layer stores bf16 (the four projections, the normalised and
rotated q, k, rho, the attention output, the layer output), must stay well
inside both element-by-element bars (FP8_LAYER_ELEM_TOL per element,
FP8_LAYER_ROW_TOL per output row) of the fp8 oracle.  Planted slips must not:
unquantised linears, one attention tile of one head copied from the tile
before it, and one head's attention output taken from its neighbour.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import layer as olayer
from local_linear_attention_streamed_b200 import synth
from _util import FP8_LAYER_ELEM_TOL, FP8_LAYER_ROW_TOL, rel_err_row, rel_err_rms, small_inputs


def _bf(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64)).float().to(torch.bfloat16).double().numpy()


def _layer_bf16_storage(x, WQ, WK, WV, WR, WO, H, slip=None):
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
    if slip == "tile":      # rows 64..127 of batch 0, head 1 copied from rows 0..63
        o = o.copy()
        o[0, 1, 64:128] = o[0, 1, 0:64]
    elif slip == "head":    # batch 1, head 0 takes head 1's output
        o = o.copy()
        o[1, 0] = o[1, 1]
    return _bf(lin(o.transpose(0, 2, 1, 3).reshape(B * N, D), WO)).reshape(B, N, D)


@pytest.mark.parametrize("B,N,D,H", [(2, 160, 256, 2), (2, 160, 256, 4), (1, 320, 512, 4)])
def test_fp8_layer_bars_are_attainable_and_discriminating(B, N, D, H):
    # The cases and seeds of tests/test_fp8_layer_gpu.py.
    _, ref = small_inputs(40 + D + H, synth.layer_specs(B, N, D), synth.BF16, device="cpu")
    args = [ref[n] for n in ("x", "WQ", "WK", "WV", "WR", "WO")]
    want = oracle.layer_fp8_ref(*args, H)
    rounded = _layer_bf16_storage(*args, H)
    assert rel_err_rms(rounded, want) <= 0.6 * FP8_LAYER_ELEM_TOL
    assert rel_err_row(rounded, want) <= 0.6 * FP8_LAYER_ROW_TOL
    unquantised = oracle.layer_fp8_ref(*args, H, linear=lambda a, W: a @ W)
    assert rel_err_row(unquantised, want) > 1.5 * FP8_LAYER_ROW_TOL
    for slip in ("tile", "head")[:B]:
        bad = _layer_bf16_storage(*args, H, slip=slip)
        assert rel_err_rms(bad, want) > 5 * FP8_LAYER_ELEM_TOL
