"""Pins of the backward-pass oracle (CPU only).

The oracle's gradients come from float64 automatic differentiation of a
vectorised statement of the forward.  They are pinned here to things other
than that statement:
  * the statement itself equals the row-by-row forward oracle (pinned in
    test_oracle.py), and a planted change to it is caught;
  * central finite differences of the row-by-row forward oracle;
  * closed forms: dV (the output is linear in V with weights that do not
    depend on V), dR (the output is linear in rho_i), the softmax-attention
    gradients when rho = 0, and a single visible key;
  * the saved statistics: equal keys give closed forms, and lse agrees with
    scipy's logsumexp;
  * the per-pair formulas the tensor-core kernels evaluate (D, F, a, dt, dl)
    reproduce the oracle's gradients.
"""
import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle
from oracle import backward as bwd


def _rand(seed, shape, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _inputs(seed, B=1, H=2, N=6, d=4, rho=0.5):
    return (_rand(seed, (B, H, N, d)), _rand(seed + 1, (B, H, N, d)), _rand(seed + 2, (B, H, N, d)),
            _rand(seed + 3, (B, H, N, d), rho), _rand(seed + 4, (B, H, N, d)))


@pytest.mark.parametrize("causal", [True, False])
def test_forward_statement_matches_row_oracle(causal):
    Q, K, V, R, _ = _inputs(1, N=9, d=8)
    got = oracle.parallax_forward_ref(Q, K, V, R, causal)
    want = oracle.prefill_ref(Q, K, V, R, causal=causal)
    assert np.max(np.abs(got - want)) < 1e-12


def _fd_grads(Q, K, V, R, dO, causal, h=1e-6):
    """Central differences of sum(prefill_ref(...) * dO) w.r.t. every input element."""
    xs = [Q.copy(), K.copy(), V.copy(), R.copy()]
    grads = []
    for a in range(4):
        g = np.zeros_like(xs[a])
        for idx in np.ndindex(xs[a].shape):
            old = xs[a][idx]
            xs[a][idx] = old + h
            fp = np.sum(oracle.prefill_ref(*xs, causal=causal) * dO)
            xs[a][idx] = old - h
            fm = np.sum(oracle.prefill_ref(*xs, causal=causal) * dO)
            xs[a][idx] = old
            g[idx] = (fp - fm) / (2 * h)
        grads.append(g)
    return grads


@pytest.mark.parametrize("causal", [True, False])
def test_backward_matches_finite_differences(causal):
    Q, K, V, R, dO = _inputs(7)
    got = oracle.parallax_backward_ref(Q, K, V, R, dO, causal)
    want = _fd_grads(Q, K, V, R, dO, causal)
    for name, g, w in zip("QKVR", got, want):
        assert np.max(np.abs(g - w)) < 1e-7 * max(1.0, np.max(np.abs(w))), name


def test_planted_mistake_in_statement_is_caught(monkeypatch):
    """A term added to the oracle's forward statement moves its gradients off
    the finite differences of the row-by-row oracle."""
    Q, K, V, R, dO = _inputs(11)
    want = _fd_grads(Q, K, V, R, dO, True)
    orig = bwd._forward_torch
    monkeypatch.setattr(bwd, "_forward_torch", lambda q, k, v, r, *a: orig(q, k, v, r, *a) + 0.05 * q * r)
    got = oracle.parallax_backward_ref(Q, K, V, R, dO, True)
    assert np.max(np.abs(got[0] - want[0])) > 1e-3


def _row_weights(Q, K, R, causal):
    """Per (b, h): softmax weights P, probe scores T = R K^T, tbar, kbar (rows)."""
    B, H, N, d = Q.shape
    out = {}
    for b in range(B):
        for h in range(H):
            P = np.zeros((N, N))
            for i in range(N):
                n = i + 1 if causal else N
                P[i, :n] = oracle.softmax_weights_row(Q[b, h, i], K[b, h, :n])
            T = R[b, h] @ K[b, h].T
            out[b, h] = (P, T, (P * T).sum(1), P @ K[b, h])
    return out


@pytest.mark.parametrize("causal", [True, False])
def test_dv_and_dr_closed_forms(causal):
    Q, K, V, R, dO = _inputs(21, N=7, d=5)
    dQ, dK, dV, dR = oracle.parallax_backward_ref(Q, K, V, R, dO, causal)
    for (b, h), (P, T, tbar, kbar) in _row_weights(Q, K, R, causal).items():
        # out_i = sum_j a_ij v_j with a_ij = p_ij (1 - t_ij + tbar_i), free of V.
        A = P * (1.0 - T + tbar[:, None])
        assert np.allclose(dV[b, h], A.T @ dO[b, h], atol=1e-12, rtol=0)
        # out_i is linear in rho_i: d/drho_i = -sum_j p_ij (dO_i . (v_j - vbar_i)) (k_j - kbar_i).
        vbar = P @ V[b, h]
        for i in range(Q.shape[2]):
            c = (V[b, h] - vbar[i]) @ dO[b, h, i]
            want = -(P[i] * c) @ (K[b, h] - kbar[i])
            assert np.allclose(dR[b, h, i], want, atol=1e-12, rtol=0)


@pytest.mark.parametrize("causal", [True, False])
def test_zero_probe_gives_softmax_attention_gradients(causal):
    Q, K, V, _, dO = _inputs(31, N=8, d=6)
    R = np.zeros_like(Q)
    dQ, dK, dV, _ = oracle.parallax_backward_ref(Q, K, V, R, dO, causal)
    d = Q.shape[-1]
    for (b, h), (P, _, _, _) in _row_weights(Q, K, R, causal).items():
        # Textbook softmax attention: dP = dO V^T, dS = P o (dP - rowsum(P o dP)).
        dP = dO[b, h] @ V[b, h].T
        dS = P * (dP - (P * dP).sum(1, keepdims=True))
        assert np.allclose(dV[b, h], P.T @ dO[b, h], atol=1e-12, rtol=0)
        assert np.allclose(dQ[b, h], dS @ K[b, h] / np.sqrt(d), atol=1e-12, rtol=0)
        assert np.allclose(dK[b, h], dS.T @ Q[b, h] / np.sqrt(d), atol=1e-12, rtol=0)


def test_single_visible_key():
    """One key: out = v_0 whatever q, k and rho are."""
    Q, K, V, R, dO = _inputs(41, N=1, d=4)
    dQ, dK, dV, dR = oracle.parallax_backward_ref(Q, K, V, R, dO, True)
    assert np.allclose(dV, dO, atol=1e-14)
    for g in (dQ, dK, dR):
        assert np.max(np.abs(g)) < 1e-14


def test_stats_closed_forms_with_equal_keys():
    B, H, N, d = 1, 2, 6, 4
    Q, _, V, R, _ = _inputs(51, B, H, N, d)
    k = _rand(57, (d,))
    K = np.broadcast_to(k, (B, H, N, d)).copy()
    vbar, lse, tbar = oracle.prefill_stats_ref(Q, K, V, R, causal=True)
    for h in range(H):
        for i in range(N):
            assert np.isclose(lse[0, h, i], np.log(i + 1) + Q[0, h, i] @ k / np.sqrt(d), atol=1e-12)
            assert np.isclose(tbar[0, h, i], R[0, h, i] @ k, atol=1e-12)
            assert np.allclose(vbar[0, h, i], V[0, h, : i + 1].mean(0), atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_stats_lse_matches_scipy(causal):
    Q, K, V, R, _ = _inputs(61, N=9, d=8)
    _, lse, _ = oracle.prefill_stats_ref(Q, K, V, R, causal)
    N, d = Q.shape[-2:]
    for h in range(Q.shape[1]):
        for i in range(N):
            n = i + 1 if causal else N
            assert np.isclose(lse[0, h, i], logsumexp(K[0, h, :n] @ Q[0, h, i] / np.sqrt(d)), atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_kernel_pair_formulas_reproduce_gradients(causal):
    """The per-pair expressions the kernels evaluate from the saved statistics:
    D = dO . vbar, F = dO . out, u = 1 - t + tbar, a = p u, dt = p (D - dA),
    dl = p (u (dA - D) + D - F); then dV = a^T dO, dR = dt K,
    dQ = dl K / sqrt(d), dK = dl^T Q / sqrt(d) + dt^T R."""
    Q, K, V, R, dO = _inputs(71, N=10, d=6)
    want = oracle.parallax_backward_ref(Q, K, V, R, dO, causal)
    out = oracle.prefill_ref(Q, K, V, R, causal=causal)
    vbar, lse, tbar = oracle.prefill_stats_ref(Q, K, V, R, causal)
    N, d = Q.shape[-2:]
    mask = np.tril(np.ones((N, N), dtype=bool)) if causal else np.ones((N, N), dtype=bool)
    for h in range(Q.shape[1]):
        q, k, v, r, g = Q[0, h], K[0, h], V[0, h], R[0, h], dO[0, h]
        P = np.where(mask, np.exp(q @ k.T / np.sqrt(d) - lse[0, h][:, None]), 0.0)
        T = r @ k.T
        dA = g @ v.T
        Dr = (g * vbar[0, h]).sum(1)[:, None]
        Fr = (g * out[0, h]).sum(1)[:, None]
        u = 1.0 - T + tbar[0, h][:, None]
        a = P * u
        dt = P * (Dr - dA)
        dl = P * (u * (dA - Dr) + Dr - Fr)
        got = (dl @ k / np.sqrt(d), dl.T @ q / np.sqrt(d) + dt.T @ r, a.T @ g, dt @ k)
        for name, x, w in zip("QKVR", got, want):
            assert np.allclose(x, w[0, h], atol=1e-11, rtol=0), name


def test_oracle_runs_on_cpu_only():
    assert not any(isinstance(x, torch.Tensor) and x.is_cuda for x in
                   oracle.parallax_backward_ref(*_inputs(81, N=3, d=2), True))


@pytest.mark.parametrize("W", [1, 3, 6])
def test_window_statement_and_gradients(W):
    """With a sliding window the statement equals the row oracle's window, and
    its gradients match central differences of that row oracle."""
    Q, K, V, R, dO = _inputs(91, N=7)
    np.testing.assert_allclose(oracle.parallax_forward_ref(Q, K, V, R, True, window=W),
                               oracle.prefill_ref(Q, K, V, R, window=W), rtol=0, atol=1e-12)
    got = oracle.parallax_backward_ref(Q, K, V, R, dO, True, window=W)
    xs = [Q.copy(), K.copy(), V.copy(), R.copy()]
    h = 1e-6
    for a in range(4):
        g = np.zeros_like(xs[a])
        for idx in np.ndindex(xs[a].shape):
            old = xs[a][idx]
            xs[a][idx] = old + h
            fp = np.sum(oracle.prefill_ref(*xs, window=W) * dO)
            xs[a][idx] = old - h
            fm = np.sum(oracle.prefill_ref(*xs, window=W) * dO)
            xs[a][idx] = old
            g[idx] = (fp - fm) / (2 * h)
        assert np.max(np.abs(got[a] - g)) < 1e-7 * max(1.0, np.max(np.abs(g)))
    vb, lse, tb = oracle.prefill_stats_ref(Q, K, V, R, True, window=W)
    if W == 1:
        np.testing.assert_allclose(vb, V, rtol=0, atol=1e-14)


def test_grouped_kv_gradients_match_finite_differences():
    """Grouped KV heads (two query heads per KV head): the gradients of K and V
    sum over the group; checked against central differences of the grouped
    row oracle."""
    rng = np.random.default_rng(101)
    B, H, Hkv, N, d = 1, 4, 2, 5, 3
    Q, R, dO = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    K, V = rng.standard_normal((B, Hkv, N, d)), rng.standard_normal((B, Hkv, N, d))
    got = oracle.parallax_backward_ref(Q, K, V, R, dO, True)
    assert got[1].shape == K.shape and got[2].shape == V.shape
    xs = [Q.copy(), K.copy(), V.copy(), R.copy()]
    h = 1e-6
    for a in range(4):
        g = np.zeros_like(xs[a])
        for idx in np.ndindex(xs[a].shape):
            old = xs[a][idx]
            xs[a][idx] = old + h
            fp = np.sum(oracle.prefill_gqa_ref(*xs, True) * dO)
            xs[a][idx] = old - h
            fm = np.sum(oracle.prefill_gqa_ref(*xs, True) * dO)
            xs[a][idx] = old
            g[idx] = (fp - fm) / (2 * h)
        assert np.max(np.abs(got[a] - g)) < 1e-7 * max(1.0, np.max(np.abs(g)))


def test_grouped_window_gradients_are_the_repeated_heads_summed():
    """Grouped KV heads under a sliding window: the gradients equal those of
    the same problem with K and V repeated over each group (one KV head per
    query head), dK and dV summed over the group's query heads."""
    rng = np.random.default_rng(102)
    B, H, Hkv, N, d, W = 1, 6, 2, 9, 3, 4
    G = H // Hkv
    Q, R, dO = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    K, V = rng.standard_normal((B, Hkv, N, d)), rng.standard_normal((B, Hkv, N, d))
    got = oracle.parallax_backward_ref(Q, K, V, R, dO, True, window=W)
    Kr, Vr = np.repeat(K, G, axis=1), np.repeat(V, G, axis=1)
    full = oracle.parallax_backward_ref(Q, Kr, Vr, R, dO, True, window=W)
    np.testing.assert_allclose(got[0], full[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[3], full[3], rtol=0, atol=1e-12)
    for a in (1, 2):
        summed = full[a].reshape(B, Hkv, G, N, d).sum(axis=2)
        np.testing.assert_allclose(got[a], summed, rtol=0, atol=1e-12)
    # The window matters here: the causal gradients differ.
    causal = oracle.parallax_backward_ref(Q, K, V, R, dO, True)
    assert np.max(np.abs(causal[1] - got[1])) > 1e-3
