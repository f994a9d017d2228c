"""Pins for the float64 oracle (CPU only).

The pages print no worked numeric example and no error bound, so the oracle
is pinned to what the mathematics and the pages' prose fix:

* hand-derived examples from the covariance form (tests/golden);
* R = 0 gives softmax attention exactly (agihunt.info summary: W_R = 0 is
  exactly softmax attention), checked against torch's float64 SDPA;
* the streamed form with one running max and one rescale factor shared by
  both branches (rainbus.top "方法步骤详情"; agihunt.info hardware paragraph)
  equals the two-pass covariance form;
* a 50-digit brute force of the raw-moment covariance matrix;
* the local-linear (weighted least squares) intercept at the solved probe
  rho* = Sigma_KK^-1 (kbar - q), the LLA special case that Parallax
  parameterises (gist.science, "Mecanismo central": rho*_i);
* closed forms (causal row 0 and row 1, identical keys) and invariants
  (weights sum to one, shift of keys, shift of values, shift of the query in
  the key-query difference, linearity in V, affinity in rho).

``test_pins_catch_mutants`` plants plausible mistakes in copies of the oracle
and checks that each is caught by at least one pin.
"""
import json
import math
import os

import mpmath
import numpy as np
import pytest
import torch

from oracle import decode_gqa_ref, decode_ref, parallax_row, prefill_ref
from oracle import layer as olayer

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------
# Independent restatements used as pins (never imported by the oracle).
# ---------------------------------------------------------------------------

def streamed_row(q, rho, K, V, block):
    """Online form: one running max m and one factor alpha rescale omega, T, O1, O2."""
    d = q.shape[0]
    m, omega, T = -math.inf, 0.0, 0.0
    O1 = np.zeros(V.shape[1])
    O2 = np.zeros(V.shape[1])
    for j0 in range(0, K.shape[0], block):
        Kb, Vb = K[j0:j0 + block], V[j0:j0 + block]
        s1 = Kb @ q / math.sqrt(d)
        t = Kb @ rho
        m_new = max(m, s1.max())
        alpha = math.exp(m - m_new) if m > -math.inf else 0.0
        w = np.exp(s1 - m_new)
        omega = alpha * omega + w.sum()
        T = alpha * T + (w * t).sum()
        O1 = alpha * O1 + w @ Vb
        O2 = alpha * O2 + (w * t) @ Vb
        m = m_new
    tbar = T / omega
    return ((1.0 + tbar) * O1 - O2) / omega


def brute_row_mp(q, rho, K, V, dps=50):
    """50-digit raw-moment form: sum_j p v - (sum_j p v k^T - vbar kbar^T) rho."""
    with mpmath.workdps(dps):
        n, d = K.shape
        dv = V.shape[1]
        qm = [mpmath.mpf(float(x)) for x in q]
        rm = [mpmath.mpf(float(x)) for x in rho]
        Km = [[mpmath.mpf(float(x)) for x in row] for row in K]
        Vm = [[mpmath.mpf(float(x)) for x in row] for row in V]
        sc = [mpmath.fsum(qm[a] * Km[j][a] for a in range(d)) / mpmath.sqrt(d) for j in range(n)]
        mx = max(sc)
        w = [mpmath.exp(s - mx) for s in sc]
        Z = mpmath.fsum(w)
        p = [x / Z for x in w]
        kbar = [mpmath.fsum(p[j] * Km[j][a] for j in range(n)) for a in range(d)]
        vbar = [mpmath.fsum(p[j] * Vm[j][c] for j in range(n)) for c in range(dv)]
        out = []
        for c in range(dv):
            # Sigma[c, a] = sum_j p_j v_jc k_ja - vbar_c kbar_a
            acc = mpmath.mpf(0)
            for a in range(d):
                sig = mpmath.fsum(p[j] * Vm[j][c] * Km[j][a] for j in range(n)) - vbar[c] * kbar[a]
                acc += sig * rm[a]
            out.append(vbar[c] - acc)
        return np.array([float(x) for x in out])


def wls_intercept(q, K, V, p):
    """Intercept of weighted least squares of v on [1, k - q] with weights p."""
    X = np.hstack([np.ones((K.shape[0], 1)), K - q[None, :]])
    sw = np.sqrt(p)[:, None]
    beta, *_ = np.linalg.lstsq(sw * X, sw * V, rcond=None)
    return beta[0]


def softmax_probs(q, K):
    s = K @ q / math.sqrt(q.shape[0])
    w = np.exp(s - s.max())
    return w / w.sum()


def solved_probe(q, K, p):
    """rho* = Sigma_KK^-1 (kbar - q) with Sigma_KK the p-weighted key covariance."""
    kbar = p @ K
    kc = K - kbar
    S = (kc * p[:, None]).T @ kc
    return np.linalg.solve(S, kbar - q)


def rows_via(row_fn, Q, K, V, R, causal=True):
    B, H, N, d = Q.shape
    out = np.empty(Q.shape[:3] + (V.shape[-1],))
    for b in range(B):
        for h in range(H):
            for i in range(N):
                n = i + 1 if causal else N
                out[b, h, i] = row_fn(Q[b, h, i], R[b, h, i], K[b, h, :n], V[b, h, :n])
    return out


# ---------------------------------------------------------------------------
# Pin checks, parameterised by the row function under test.
# ---------------------------------------------------------------------------

def pin_golden(row_fn):
    with open(GOLDEN) as f:
        data = json.load(f)
    for case in data["cases"]:
        if case.get("q_expr") == "sqrt2_ln3_first":
            q = np.array([math.sqrt(2.0) * math.log(3.0), 0.0])
        else:
            q = np.array(case["q"], dtype=np.float64)
        K = np.array(case["K"], dtype=np.float64)
        V = np.array(case["V"], dtype=np.float64)
        rho = np.array(case["rho"], dtype=np.float64)
        got = row_fn(q, rho, K, V)
        np.testing.assert_allclose(got, case["expected"], rtol=0, atol=1e-13, err_msg=case["name"])
        # Weights s_j: the output for V = identity.
        sw = row_fn(q, rho, K, np.eye(K.shape[0]))
        np.testing.assert_allclose(sw, case["weights"], rtol=0, atol=1e-13, err_msg=case["name"])


def pin_softmax_when_r_zero(row_fn):
    rng = _rng(1)
    B, H, N, d = 1, 2, 24, 8
    Q, K, V = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    R = np.zeros_like(Q)
    for causal in (True, False):
        got = rows_via(row_fn, Q, K, V, R, causal)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(Q), torch.from_numpy(K), torch.from_numpy(V), is_causal=causal).numpy()
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-13)


def pin_streamed_equals_covariance(row_fn):
    rng = _rng(2)
    for (n, d) in [(1, 4), (7, 4), (33, 16), (64, 8)]:
        q, rho = rng.standard_normal(d), 0.5 * rng.standard_normal(d)
        K, V = rng.standard_normal((n, d)), rng.standard_normal((n, d))
        got = row_fn(q, rho, K, V)
        for blk in (1, 16, n):
            np.testing.assert_allclose(got, streamed_row(q, rho, K, V, blk), rtol=0, atol=1e-12)


def pin_brute_force(row_fn):
    rng = _rng(3)
    for (n, d, dv) in [(1, 3, 2), (3, 3, 3), (5, 4, 2), (8, 4, 5)]:
        q, rho = rng.standard_normal(d), rng.standard_normal(d)
        K, V = rng.standard_normal((n, d)), rng.standard_normal((n, dv))
        np.testing.assert_allclose(row_fn(q, rho, K, V), brute_row_mp(q, rho, K, V), rtol=0, atol=1e-13)


def pin_wls_intercept(row_fn):
    rng = _rng(4)
    for (n, d, dv) in [(6, 2, 3), (8, 3, 2), (12, 4, 4)]:
        q = rng.standard_normal(d)
        K, V = rng.standard_normal((n, d)), rng.standard_normal((n, dv))
        p = softmax_probs(q, K)
        rho = solved_probe(q, K, p)
        np.testing.assert_allclose(row_fn(q, rho, K, V), wls_intercept(q, K, V, p), rtol=0, atol=1e-10)


def pin_closed_forms(row_fn):
    rng = _rng(5)
    d = 6
    K, V = rng.standard_normal((2, d)), rng.standard_normal((2, d))
    q, rho = rng.standard_normal(d), rng.standard_normal(d)
    # A single visible key: out = v_0 (causal row 0).
    np.testing.assert_allclose(row_fn(q, rho, K[:1], V[:1]), V[0], rtol=0, atol=1e-15)
    # Two visible keys: out = p0 v0 + p1 v1 - p0 p1 (v1 - v0) ((k1 - k0).rho).
    p = softmax_probs(q, K)
    exp = p[0] * V[0] + p[1] * V[1] - p[0] * p[1] * (V[1] - V[0]) * ((K[1] - K[0]) @ rho)
    np.testing.assert_allclose(row_fn(q, rho, K, V), exp, rtol=0, atol=1e-13)
    # Identical keys: uniform weights, zero key spread: out = mean of the values.
    Kc = np.repeat(rng.standard_normal((1, d)), 5, axis=0)
    Vc = rng.standard_normal((5, d))
    np.testing.assert_allclose(row_fn(q, rho, Kc, Vc), Vc.mean(axis=0), rtol=0, atol=1e-14)


def pin_invariants(row_fn):
    rng = _rng(6)
    n, d = 20, 8
    q, rho = rng.standard_normal(d), rng.standard_normal(d)
    K, V = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    base = row_fn(q, rho, K, V)
    c = rng.standard_normal(d)
    # Weights sum to one: V = all ones gives ones.
    np.testing.assert_allclose(row_fn(q, rho, K, np.ones((n, 3))), np.ones(3), rtol=0, atol=1e-13)
    # Value shift moves the output by the shift.
    np.testing.assert_allclose(row_fn(q, rho, K, V + c), base + c, rtol=0, atol=1e-12)
    # Key shift by a common vector changes nothing.
    np.testing.assert_allclose(row_fn(q, rho, K + c, V), base, rtol=0, atol=1e-12)
    # Linear in V, affine in rho.
    V2 = rng.standard_normal((n, d))
    np.testing.assert_allclose(row_fn(q, rho, K, 2.0 * V - 3.0 * V2),
                               2.0 * base - 3.0 * row_fn(q, rho, K, V2), rtol=0, atol=1e-12)
    r2 = rng.standard_normal(d)
    o0 = row_fn(q, np.zeros(d), K, V)
    lhs = row_fn(q, 0.3 * rho + 0.7 * r2, K, V)
    rhs = 0.3 * base + 0.7 * row_fn(q, r2, K, V) + (1 - 0.3 - 0.7) * o0
    np.testing.assert_allclose(lhs, rhs, rtol=0, atol=1e-12)
    # Weights may be negative (the pages: scores may go below zero or far above one).
    sw = row_fn(q, 3.0 * rho, K, np.eye(n))
    assert sw.min() < 0.0


def pin_query_shift(row_fn):
    """The probe term of z_ij = k_j - q_i: rho . (k_j - q_i - c) gives the same output."""
    rng = _rng(7)
    n, d = 17, 8
    q, rho = rng.standard_normal(d), rng.standard_normal(d)
    K, V = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    p = softmax_probs(q, K)
    for shift in (np.zeros(d), q, q + rng.standard_normal(d)):
        Z = K - shift[None, :]
        t = Z @ rho
        tbar = p @ t
        s = p * (1.0 - t + tbar)
        np.testing.assert_allclose(row_fn(q, rho, K, V), s @ V, rtol=0, atol=1e-12)


ROW_PINS = [pin_golden, pin_softmax_when_r_zero, pin_streamed_equals_covariance, pin_brute_force,
            pin_wls_intercept, pin_closed_forms, pin_invariants, pin_query_shift]


@pytest.mark.parametrize("pin", ROW_PINS, ids=lambda f: f.__name__)
def test_oracle_row_pins(pin):
    pin(parallax_row)


# ---------------------------------------------------------------------------
# Mutants: every plausible slip must trip at least one pin.
# ---------------------------------------------------------------------------

def _mut_sign(q, rho, K, V):
    p = softmax_probs(q, K)
    kbar, vbar = p @ K, p @ V
    return vbar + (V - vbar).T @ (p * ((K - kbar) @ rho))


def _mut_unweighted_means(q, rho, K, V):
    p = softmax_probs(q, K)
    ku, vu = K.mean(axis=0), V.mean(axis=0)
    return p @ V - (V - vu).T @ (p * ((K - ku) @ rho))


def _mut_raw_second_moment(q, rho, K, V):
    p = softmax_probs(q, K)
    return p @ V - V.T @ (p * (K @ rho))


def _mut_scaled_probe(q, rho, K, V):
    p = softmax_probs(q, K)
    kbar, vbar = p @ K, p @ V
    return vbar - (V - vbar).T @ (p * ((K - kbar) @ rho)) / math.sqrt(q.shape[0])


def _mut_unscaled_scores(q, rho, K, V):
    s = K @ q
    w = np.exp(s - s.max())
    p = w / w.sum()
    kbar, vbar = p @ K, p @ V
    return vbar - (V - vbar).T @ (p * ((K - kbar) @ rho))


def _mut_probe_uses_query(q, rho, K, V):
    p = softmax_probs(q, K)
    kbar, vbar = p @ K, p @ V
    return vbar - (V - vbar).T @ (p * ((K - kbar) @ q))


def _mut_unnormalised_weights(q, rho, K, V):
    s = K @ q / math.sqrt(q.shape[0])
    p = np.exp(s - s.max())
    kbar, vbar = p @ K, p @ V
    return vbar - (V - vbar).T @ (p * ((K - kbar) @ rho))


# (Centring only one factor of the covariance, or centring one factor by any
# constant, is not a mistake: sum_j p_j (x_j - xbar) = 0 makes the second
# centring redundant, so no pin can or should tell those forms apart.)
MUTANTS = [_mut_sign, _mut_unweighted_means, _mut_raw_second_moment, _mut_scaled_probe,
           _mut_unscaled_scores, _mut_probe_uses_query, _mut_unnormalised_weights]


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda f: f.__name__)
def test_pins_catch_mutants(mutant):
    caught = []
    for pin in ROW_PINS:
        try:
            pin(mutant)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught {mutant.__name__}"


def test_prefill_and_decode_conventions():
    """Causal row i sees keys 0..i; a decode query at length n equals prefill row n-1."""
    rng = _rng(8)
    B, H, N, d = 2, 2, 9, 4
    Q, K, V = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    R = 0.3 * rng.standard_normal((B, H, N, d))
    full = prefill_ref(Q, K, V, R, causal=True)
    np.testing.assert_allclose(full[:, :, 0], V[:, :, 0], rtol=0, atol=1e-15)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q), torch.from_numpy(K), torch.from_numpy(V), is_causal=True).numpy()
    np.testing.assert_allclose(prefill_ref(Q, K, V, 0 * R, causal=True), ref, rtol=0, atol=1e-13)
    picked = prefill_ref(Q, K, V, R, causal=False, rows=[(1, 0, 3), (0, 1, 8)])
    np.testing.assert_allclose(picked[1], full[0, 1, 8], rtol=0, atol=1e-14)
    seqlens = np.array([5, 9])
    dec = decode_ref(Q[:, :, 0] * 0 + Q[np.arange(B), :, seqlens - 1], R[np.arange(B), :, seqlens - 1],
                     K, V, seqlens)
    for b in range(B):
        np.testing.assert_allclose(dec[b], full[b, :, seqlens[b] - 1], rtol=0, atol=1e-14)


def test_decode_gqa_pins():
    """Grouped KV heads: query head h reads KV head h // G.

    Pinned to the MHA oracle on the KV heads repeated G times (np.repeat puts
    the copies of one KV head next to each other), which a head map of
    h % Hkv would fail; G = 1 is the MHA oracle itself; heads of one group
    with equal q and rho give equal outputs.
    """
    rng = _rng(21)
    B, Hkv, G, L, d = 2, 3, 4, 11, 8
    H = Hkv * G
    q = rng.standard_normal((B, H, d))
    r = 0.3 * rng.standard_normal((B, H, d))
    Kc, Vc = rng.standard_normal((B, Hkv, L, d)), rng.standard_normal((B, Hkv, L, d))
    seqlens = np.array([7, 11])
    got = decode_gqa_ref(q, r, Kc, Vc, seqlens)
    want = decode_ref(q, r, np.repeat(Kc, G, axis=1), np.repeat(Vc, G, axis=1), seqlens)
    np.testing.assert_allclose(got, want, rtol=0, atol=0)
    wrong = decode_ref(q, r, np.tile(Kc, (1, G, 1, 1)), np.tile(Vc, (1, G, 1, 1)), seqlens)
    assert np.abs(got - wrong).max() > 1e-3
    np.testing.assert_allclose(decode_gqa_ref(q[:, :Hkv], r[:, :Hkv], Kc, Vc, seqlens),
                               decode_ref(q[:, :Hkv], r[:, :Hkv], Kc, Vc, seqlens), rtol=0, atol=0)
    q2, r2 = q.copy(), r.copy()
    q2[:, 5], r2[:, 5] = q2[:, 4], r2[:, 4]  # heads 4 and 5 share KV head 1
    same = decode_gqa_ref(q2, r2, Kc, Vc, seqlens)
    np.testing.assert_allclose(same[:, 5], same[:, 4], rtol=0, atol=0)
    picked = decode_gqa_ref(q, r, Kc, Vc, seqlens, units=[(1, 7), (0, 0)])
    np.testing.assert_allclose(picked, np.stack([got[1, 7], got[0, 0]]), rtol=0, atol=0)


# ---------------------------------------------------------------------------
# Layer pieces: RMSNorm and RoPE.
# ---------------------------------------------------------------------------

def test_rmsnorm_pins():
    rng = _rng(9)
    x = rng.standard_normal((5, 16))
    y = olayer.rmsnorm(x, eps=0.0)
    np.testing.assert_allclose(np.sqrt((y * y).mean(-1)), 1.0, rtol=0, atol=1e-14)
    np.testing.assert_allclose(olayer.rmsnorm(7.5 * x, eps=0.0), y, rtol=0, atol=1e-14)
    # With eps the RMS is sqrt(ms / (ms + eps)).
    ms = (x * x).mean(-1)
    ye = olayer.rmsnorm(x, eps=0.5)
    np.testing.assert_allclose(np.sqrt((ye * ye).mean(-1)), np.sqrt(ms / (ms + 0.5)), rtol=1e-14)


def test_rope_pins():
    rng = _rng(10)
    d = 16
    x = rng.standard_normal((4, d))
    np.testing.assert_allclose(olayer.rope(x, np.zeros(4)), x, rtol=0, atol=0)
    pos = np.array([0, 3, 17, 1000])
    y = olayer.rope(x, pos)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-14)
    # Complex form: (x_k + i x_{k+d/2}) * exp(i pos theta_k), theta_k = 10000^(-2k/d).
    half = d // 2
    theta = 10000.0 ** (-2.0 * np.arange(half) / d)
    z = (x[:, :half] + 1j * x[:, half:]) * np.exp(1j * pos[:, None] * theta[None, :])
    np.testing.assert_allclose(y, np.concatenate([z.real, z.imag], axis=-1), rtol=0, atol=1e-13)
    # Relative position: <rope(a, m), rope(b, n)> depends on m - n only.
    a, b = rng.standard_normal(d), rng.standard_normal(d)
    d1 = olayer.rope(a, np.array(7)) @ olayer.rope(b, np.array(2))
    d2 = olayer.rope(a, np.array(105)) @ olayer.rope(b, np.array(100))
    assert abs(d1 - d2) < 1e-12


def test_layer_softmax_when_wr_zero():
    """W_R = 0 makes the layer softmax attention (checked against torch SDPA)."""
    rng = _rng(11)
    B, N, D, H = 2, 12, 32, 4
    d = D // H
    x = rng.standard_normal((B, N, D))
    WQ, WK, WV, WO = (rng.standard_normal((D, D)) / math.sqrt(D) for _ in range(4))
    WR = np.zeros((D, D))
    rows = [(0, 0), (0, 5), (1, 11), (1, 7)]
    got = olayer.layer_rows_ref(x, WQ, WK, WV, WR, WO, H, rows)
    pos = np.arange(N)

    def heads(W):
        return (x @ W).reshape(B, N, H, d).transpose(0, 2, 1, 3)

    def nr(y):
        ms = (y * y).mean(-1, keepdims=True)
        y = y / np.sqrt(ms + 1e-6)
        half = d // 2
        th = 10000.0 ** (-2.0 * np.arange(half) / d)
        z = (y[..., :half] + 1j * y[..., half:]) * np.exp(1j * pos[None, None, :, None] * th)
        return np.concatenate([z.real, z.imag], axis=-1)

    q, k, v = nr(heads(WQ)), nr(heads(WK)), heads(WV)
    o = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=True).numpy()
    y = o.transpose(0, 2, 1, 3).reshape(B, N, D) @ WO
    for idx, (b, t) in enumerate(rows):
        np.testing.assert_allclose(got[idx], y[b, t], rtol=0, atol=1e-12)


def test_layer_row_matches_head_oracle():
    """A layer row is W_O applied to the per-head oracle on normalised, rotated q, k, rho."""
    rng = _rng(12)
    B, N, D, H = 1, 10, 16, 2
    x = rng.standard_normal((B, N, D))
    W = [rng.standard_normal((D, D)) / math.sqrt(D) for _ in range(5)]
    got = olayer.layer_rows_ref(x, *W, H, [(0, 9)])
    q = olayer.qkr_norm_rope_ref(x, W[0], H)
    k = olayer.qkr_norm_rope_ref(x, W[1], H)
    r = olayer.qkr_norm_rope_ref(x, W[3], H)
    v = (x @ W[2]).reshape(B, N, H, D // H).transpose(0, 2, 1, 3)
    o = prefill_ref(q, k, v, r, causal=True)
    y = o.transpose(0, 2, 1, 3).reshape(B, N, D) @ W[4]
    np.testing.assert_allclose(got[0], y[0, 9], rtol=0, atol=1e-12)


def test_prefill_gqa_pins():
    """Grouped KV heads in the prefill: equal to the ungrouped oracle with each
    KV head repeated for its query heads (np.repeat, not the oracle's index
    map), G = 1 is the ungrouped prefill, and swapping two KV heads permutes
    the output groups."""
    from oracle import prefill_gqa_ref
    rng = _rng(30)
    B, H, Hkv, N, d = 2, 6, 2, 9, 4
    Q, R = rng.standard_normal((B, H, N, d)), rng.standard_normal((B, H, N, d))
    K, V = rng.standard_normal((B, Hkv, N, d)), rng.standard_normal((B, Hkv, N, d))
    G = H // Hkv
    for causal in (True, False):
        want = prefill_ref(Q, np.repeat(K, G, axis=1), np.repeat(V, G, axis=1), R, causal=causal)
        np.testing.assert_allclose(prefill_gqa_ref(Q, K, V, R, causal), want, rtol=0, atol=1e-13)
    K1, V1 = rng.standard_normal((B, H, N, d)), rng.standard_normal((B, H, N, d))
    np.testing.assert_allclose(prefill_gqa_ref(Q, K1, V1, R), prefill_ref(Q, K1, V1, R), rtol=0, atol=0)
    # Reversing the KV heads hands the first group of query heads the last KV head.
    sw = prefill_gqa_ref(Q, K[:, ::-1].copy(), V[:, ::-1].copy(), R)
    np.testing.assert_allclose(sw[:, :G], prefill_gqa_ref(Q[:, :G], K[:, -1:], V[:, -1:], R[:, :G]),
                               rtol=0, atol=1e-13)
