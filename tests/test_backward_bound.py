"""The backward parity bars are attainable and still discriminating (CPU only).

The float64 gradients (oracle) recomputed with bf16 rounding at exactly the
points where the CUDA backward rounds -- the output used for F = dO . out,
the per-pair weights a, dl/sqrt(d) and dt before their MMAs, and the stored
gradients -- with or without the training forward's own rounding (its value
MMAs take bf16 weights, so the saved vbar and out carry it), must stay inside
GRAD_TOL (relative Frobenius error) and GRAD_MAX_TOL (largest elementwise
error).  Plausible slips (the mean probe score left out of u, or D used where
D - F belongs) must land far outside GRAD_TOL.
"""
import numpy as np
import pytest
import torch

import oracle
from local_linear_attention_streamed_b200 import synth
from _util import GRAD_MAX_TOL, GRAD_TOL, rel_err_elem, rel_err_fro, small_inputs


def _bf(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64)).float().to(torch.bfloat16).double().numpy()


def _kernel_rounding(ref, causal, slip=None, forward_rounding=False):
    """Gradients from the per-pair expressions, rounded where the kernels round
    (and, with forward_rounding, vbar and out from bf16-rounded weights: bf16(p)
    for the mean, bf16(p (t - tbar)) for the centred correction)."""
    Q, K, V, R, dO = (ref[n] for n in ("Q", "K", "V", "R", "dO"))
    out_all = _bf(oracle.prefill_ref(Q, K, V, R, causal=causal))
    vbar_all, lse, tbar = oracle.prefill_stats_ref(Q, K, V, R, causal)
    B, H, N, d = Q.shape
    mask = np.tril(np.ones((N, N), dtype=bool)) if causal else np.ones((N, N), dtype=bool)
    res = [np.zeros_like(Q) for _ in range(4)]
    for b in range(B):
        for h in range(H):
            q, k, v, r, g = Q[b, h], K[b, h], V[b, h], R[b, h], dO[b, h]
            P = np.where(mask, np.exp(q @ k.T / np.sqrt(d) - lse[b, h][:, None]), 0.0)
            T = r @ k.T
            dA = g @ v.T
            vbar, out = vbar_all[b, h], out_all[b, h]
            if forward_rounding:
                vbar = _bf(P) @ v
                out = _bf(vbar - _bf(P * (T - tbar[b, h][:, None])) @ v)
            D = (g * vbar).sum(1)[:, None]
            F = (g * out).sum(1)[:, None]
            u = 1.0 - T + (0.0 if slip == "no_tbar" else tbar[b, h][:, None])
            c = D if slip == "D_for_D_minus_F" else D - F
            a, dt, dl = _bf(P * u), _bf(P * (D - dA)), _bf(P * (u * (dA - D) + c) / np.sqrt(d))
            res[0][b, h], res[1][b, h] = dl @ k, dl.T @ q + dt.T @ r
            res[2][b, h], res[3][b, h] = a.T @ g, dt @ k
    return [_bf(x) for x in res]


CASES = [(128, 128, True), (200, 128, True), (192, 128, False), (384, 128, True), (256, 64, True),
         (130, 64, False), (1024, 128, True)]


@pytest.mark.parametrize("N,d,causal", CASES)
@pytest.mark.parametrize("forward_rounding", [False, True])
def test_kernel_rounding_stays_inside_bar(N, d, causal, forward_rounding):
    H = 1 if N > 512 else 2
    _, ref = small_inputs(900 + N + d, synth.backward_specs(1, H, N, d), synth.BF16, device="cpu")
    want = oracle.parallax_backward_ref(ref["Q"], ref["K"], ref["V"], ref["R"], ref["dO"], causal)
    got = _kernel_rounding(ref, causal, forward_rounding=forward_rounding)
    fro = [rel_err_fro(g, w) for g, w in zip(got, want)]
    assert max(fro) <= 0.3 * GRAD_TOL, fro
    emax = [rel_err_elem(g, w) for g, w in zip(got, want)]
    assert max(emax) <= 0.6 * GRAD_MAX_TOL, emax


@pytest.mark.parametrize("slip", ["no_tbar", "D_for_D_minus_F"])
def test_slips_fail_the_bar(slip):
    _, ref = small_inputs(950, synth.backward_specs(1, 2, 160, 128), synth.BF16, device="cpu")
    want = oracle.parallax_backward_ref(ref["Q"], ref["K"], ref["V"], ref["R"], ref["dO"], True)
    got = _kernel_rounding(ref, True, slip=slip)
    assert max(rel_err_fro(g, w) for g, w in zip(got, want)) > 5 * GRAD_TOL
