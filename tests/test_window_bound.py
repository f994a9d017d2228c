"""The sliding-window prefill's centring rules, emulated in float64 (CPU only).

The tensor-core prefill rounds two operands per key to bf16 before its value
MMAs: w and w (t - c), with c a per-row centre of the probe scores t.  How
well c tracks the running softmax mean of t decides how much that rounding is
amplified in out = ((1 + T/omega) O1 - O2) / omega.  This test replays the
kernel's per-row block arithmetic (64-key blocks at absolute positions, the
lazy max raised only by more than 2^8, the centre set by the row's first block
with weight and moved on drift, bf16 rounding of both operands) with float64
everywhere else, and checks:
  * with the windowed kernel's rules (a forced re-centre on the row's second
    block when its window starts inside the previous block; drift threshold
    0.5 below 256 keys) a 37-key window stays inside the bf16 bar;
  * with the causal kernel's rules (threshold 2, no forced re-centre) it does
    not: the reason the windowed variant has its own rules.
The same emulation reproduces the GPU's error on these inputs to four digits.
"""
import numpy as np
import torch

import oracle
from local_linear_attention_streamed_b200 import synth
from _util import BF16_TOL, rel_err_rms, small_inputs


def _bf(a):
    return torch.from_numpy(np.atleast_1d(np.asarray(a, dtype=np.float64))).float().to(torch.bfloat16).double().numpy()


def _f32(a):
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def _row(q, r, K, V, i, W, theta, force_second, BN=64, tau=8.0):
    d = q.shape[0]
    sc = 1.4426950408889634 / np.sqrt(d)
    lo = max(0, i - W + 1)
    m, om, T, c = -np.inf, 0.0, 0.0, 0.0
    O1 = np.zeros(V.shape[1])
    O2 = np.zeros(V.shape[1])
    for kb in range(lo // BN * BN, i + 1, BN):
        Kb, Vb = K[kb:kb + BN], V[kb:kb + BN]
        keys = np.arange(kb, kb + Kb.shape[0])
        vis = (keys >= lo) & (keys <= i)
        s = np.where(vis, _f32(Kb @ q) * sc, -np.inf)
        t = _f32(Kb @ r)
        mx = s.max()
        if mx > m + tau:
            a = 2.0 ** (m - mx) if m > -np.inf else 0.0
            m, om, T, O1, O2 = mx, om * a, T * a, O1 * a, O2 * a
        w = np.where(vis, 2.0 ** (s - (0.0 if m == -np.inf else m)), 0.0)
        wb, tb = w.sum(), (w * (t - c)).sum()
        Wp, Wn = om, om + wb
        second = force_second and kb - BN < lo < kb
        if Wn > 0 and (Wp == 0 or second or abs((T + tb) / Wn) > theta):
            delta = (T + tb) / Wn
            c += delta
            O2 -= delta * O1
            T -= delta * om
            tb -= delta * wb
        om += wb
        T += tb
        O1 += _bf(w) @ Vb
        O2 += _bf(w * (t - c)) @ Vb
    return _bf(((1 + T / om) * O1 - O2) / om)


def _emulate(ref, W, theta, force_second):
    Q, K, V, R = (ref[n] for n in ("Q", "K", "V", "R"))
    H, N = Q.shape[1], Q.shape[2]
    out = np.zeros(Q.shape)
    for h in range(H):
        for i in range(N):
            out[0, h, i] = _row(Q[0, h, i], R[0, h, i], K[0, h], V[0, h], i, W, theta, force_second)
    return out


def test_window_rules_meet_the_bar_where_causal_rules_do_not():
    W, N = 37, 300
    _, ref = small_inputs(700 + N + W, synth.prefill_specs(1, 3, N, 128), synth.BF16, device="cpu")
    want = oracle.prefill_ref(ref["Q"], ref["K"], ref["V"], ref["R"], window=W)
    window_rules = rel_err_rms(_emulate(ref, W, 0.5, True), want)
    causal_rules = rel_err_rms(_emulate(ref, W, 2.0, False), want)
    assert window_rules <= 0.85 * BF16_TOL, window_rules
    assert causal_rules > BF16_TOL, causal_rules
