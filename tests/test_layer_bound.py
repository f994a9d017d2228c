"""The layer parity bar is attainable and still discriminating (CPU only).

The float64 layer oracle rounded to bf16 at the five points where the CUDA
layer stores bf16 (projections, normalised and rotated q/k/rho, head-split v,
attention output, layer output) must stay inside LAYER_TOL; a layer with a
plausible slip (RMSNorm left out of rho, or RoPE left out of k) must not.
"""
import numpy as np
import torch

import oracle
from local_linear_attention_streamed_b200 import synth
from _util import LAYER_TOL, rel_err_rms, small_inputs

B, N, D, H = 2, 160, 256, 2
d = D // H


def _bf(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64)).float().to(torch.bfloat16).double().numpy()


def _heads(y):
    return y.reshape(B, N, H, d).transpose(0, 2, 1, 3)


def _pipeline(ref, rnd, norm_r=True, rope_k=True):
    x = ref["x"]
    pos = np.arange(N)[None, None, :]

    def nr(W, norm=True, rot=True):
        y = _heads(rnd(x @ ref[W]))
        if norm:
            y = oracle.rmsnorm(y)
        if rot:
            y = oracle.rope(y, pos)
        return rnd(y)

    q, k, r = nr("WQ"), nr("WK", rot=rope_k), nr("WR", norm=norm_r)
    v = rnd(_heads(x @ ref["WV"]))
    o = rnd(oracle.prefill_ref(q, k, v, r, causal=True))
    return rnd(o.transpose(0, 2, 1, 3).reshape(B, N, D) @ ref["WO"])


def test_layer_bar_attainable_and_discriminating():
    specs = synth.layer_specs(B, N, D)
    _, ref = small_inputs(1005, specs, synth.BF16, device="cpu")
    rows = [(b, t) for b in range(B) for t in range(N)]
    want = oracle.layer_rows_ref(ref["x"], ref["WQ"], ref["WK"], ref["WV"], ref["WR"], ref["WO"], H,
                                 rows).reshape(B, N, D)
    exact = _pipeline(ref, lambda a: a)
    assert rel_err_rms(exact, want) < 1e-10
    rounded = _pipeline(ref, _bf)
    assert rel_err_rms(rounded, want) <= 0.9 * LAYER_TOL
    assert rel_err_rms(_pipeline(ref, _bf, norm_r=False), want) > 2 * LAYER_TOL
    assert rel_err_rms(_pipeline(ref, _bf, rope_k=False), want) > 2 * LAYER_TOL
