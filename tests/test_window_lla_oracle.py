"""Pins of the oracle's sliding-window reading and of the exact-LLA extension (CPU only).

Sliding window (W keys: query i sees keys max(0, i - W + 1)..i; a decode
query at length n sees the last W keys):
  * W >= N is the causal prefill; W = 1 gives out_i = v_i exactly;
  * row i equals the last row of the causal prefill of the W-key subsequence
    that ends at i (a different path through the oracle);
  * the decode window at length n equals the prefill window's row n - 1;
  * an off-by-one window planted in the oracle is caught.

Exact LLA (the local-linear estimator whose per-query solve Parallax
parameterises; gist.science, "Mecanismo central"):
  * the Parallax form at the solved probe rho* equals the ridge-regression
    intercept, for several regularisations lambda;
  * with lambda = 0 and more keys than dimensions, values that are an affine
    function of the keys are reproduced exactly at the query (the defining
    property of a local-linear fit), which softmax attention does not do;
  * lambda -> infinity gives softmax attention (rho* -> 0).

Block sparsity (a mask over 128-query tiles and 64-key blocks): all blocks
active is causal, diagonal blocks only is a per-tile causal prefill, and rows
of a strided pattern see exactly the causal keys of their active blocks.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import parallax as opar


def _rng(seed):
    return np.random.default_rng(seed)


def _inputs(seed, B=1, H=2, N=11, d=4):
    rng = _rng(seed)
    return tuple(rng.standard_normal((B, H, N, d)) for _ in range(3)) + (0.5 * rng.standard_normal((B, H, N, d)),)


def test_window_covering_everything_is_causal():
    Q, K, V, R = _inputs(1)
    N = Q.shape[2]
    causal = oracle.prefill_ref(Q, K, V, R, causal=True)
    for W in (N, N + 5):
        np.testing.assert_allclose(oracle.prefill_ref(Q, K, V, R, window=W), causal, rtol=0, atol=0)


def test_window_of_one_returns_own_value():
    Q, K, V, R = _inputs(2)
    np.testing.assert_allclose(oracle.prefill_ref(Q, K, V, R, window=1), V, rtol=0, atol=1e-14)


@pytest.mark.parametrize("W", [2, 3, 5])
def test_window_row_is_last_row_of_subsequence(W):
    Q, K, V, R = _inputs(3)
    got = oracle.prefill_ref(Q, K, V, R, window=W)
    N = Q.shape[2]
    for i in range(N):
        lo = max(0, i - W + 1)
        sub = [x[:, :, lo:i + 1] for x in (Q, K, V, R)]
        want = oracle.prefill_ref(*sub, causal=True)[:, :, -1]
        np.testing.assert_allclose(got[:, :, i], want, rtol=0, atol=1e-13)


def test_decode_window_matches_prefill_window():
    Q, K, V, R = _inputs(4, B=2, H=2, N=9)
    W = 4
    pre = oracle.prefill_ref(Q, K, V, R, window=W)
    for n in (1, 3, 4, 9):
        seqlens = np.array([n, n])
        got = oracle.decode_ref(Q[:, :, n - 1], R[:, :, n - 1], K, V, seqlens, window=W)
        np.testing.assert_allclose(got, pre[:, :, n - 1], rtol=0, atol=1e-13)


def test_off_by_one_window_is_caught(monkeypatch):
    Q, K, V, R = _inputs(5)
    orig = opar.visible_keys

    def off_by_one(i, N, causal, window=None):
        lo, hi = orig(i, N, causal, window)
        return (max(0, lo - 1), hi) if window is not None else (lo, hi)

    monkeypatch.setattr(opar, "visible_keys", off_by_one)
    got = oracle.prefill_ref(Q, K, V, R, window=1)
    assert np.max(np.abs(got - V)) > 1e-3


@pytest.mark.parametrize("lam", [0.0, 0.1, 3.0])
def test_parallax_at_solved_probe_is_lla(lam):
    rng = _rng(10)
    n, d = 14, 5
    q, K, V = rng.standard_normal(d), rng.standard_normal((n, d)), rng.standard_normal((n, 3))
    rho = oracle.lla_probe(q, K, lam)
    np.testing.assert_allclose(oracle.parallax_row(q, rho, K, V), oracle.lla_row(q, K, V, lam),
                               rtol=0, atol=1e-11)


def test_lla_reproduces_affine_values_exactly():
    rng = _rng(11)
    n, d = 16, 4
    q, K = rng.standard_normal(d), rng.standard_normal((n, d))
    A, c = rng.standard_normal((d, 3)), rng.standard_normal(3)
    V = K @ A + c
    want = q @ A + c
    np.testing.assert_allclose(oracle.lla_row(q, K, V, 0.0), want, rtol=0, atol=1e-11)
    rho = oracle.lla_probe(q, K, 0.0)
    np.testing.assert_allclose(oracle.parallax_row(q, rho, K, V), want, rtol=0, atol=1e-10)
    # Softmax attention (rho = 0) does not: it returns the weighted mean.
    assert np.max(np.abs(oracle.parallax_row(q, np.zeros(d), K, V) - want)) > 1e-2


def test_lla_with_infinite_regularisation_is_softmax():
    rng = _rng(12)
    n, d = 9, 4
    q, K, V = rng.standard_normal(d), rng.standard_normal((n, d)), rng.standard_normal((n, 3))
    np.testing.assert_allclose(oracle.lla_row(q, K, V, 1e12), oracle.parallax_row(q, np.zeros(d), K, V),
                               rtol=0, atol=1e-9)
    assert np.max(np.abs(oracle.lla_probe(q, K, 1e12))) < 1e-9


def test_lla_prefill_ref_shapes_and_rows():
    Q, K, V, _ = _inputs(13, N=7, d=3)
    out, Rs = oracle.lla_prefill_ref(Q, K, V, 0.5, causal=True)
    assert out.shape == V.shape and Rs.shape == Q.shape
    np.testing.assert_allclose(out, oracle.prefill_ref(Q, K, V, Rs, causal=True), rtol=0, atol=1e-11)


# ---------------------------------------------------------------------------
# Block-sparse reading: mask over (128-query tile, 64-key block) pairs.
# ---------------------------------------------------------------------------

def _sparse_inputs(seed, N=300, d=4):
    rng = _rng(seed)
    return tuple(rng.standard_normal((1, 2, N, d)) for _ in range(3)) + (0.5 * rng.standard_normal((1, 2, N, d)),)


def _mask(N, active):
    nt, nkb = (N + 127) // 128, (N + 63) // 64
    m = np.zeros((nt, nkb), dtype=bool)
    for t in range(nt):
        for kb in range(nkb):
            m[t, kb] = active(t, kb)
    return m


def test_block_sparse_all_active_is_causal():
    Q, K, V, R = _sparse_inputs(20)
    m = _mask(300, lambda t, kb: True)
    np.testing.assert_allclose(oracle.prefill_block_sparse_ref(Q, K, V, R, m),
                               oracle.prefill_ref(Q, K, V, R, causal=True), rtol=0, atol=1e-13)


def test_block_sparse_diagonal_blocks_only_is_a_per_tile_prefill():
    """Only each tile's own two key blocks: every tile is an independent causal
    prefill of its 128 positions."""
    Q, K, V, R = _sparse_inputs(21)
    N = 300
    m = _mask(N, lambda t, kb: kb // 2 == t)
    got = oracle.prefill_block_sparse_ref(Q, K, V, R, m)
    for t in range(3):
        lo, hi = 128 * t, min(N, 128 * t + 128)
        sub = [x[:, :, lo:hi] for x in (Q, K, V, R)]
        np.testing.assert_allclose(got[:, :, lo:hi], oracle.prefill_ref(*sub, causal=True), rtol=0, atol=1e-13)


def test_block_sparse_rows_see_exactly_their_blocks():
    """A strided pattern: each visible-key set is the causal keys of the active blocks."""
    Q, K, V, R = _sparse_inputs(22)
    m = _mask(300, lambda t, kb: kb // 2 == t or kb % 3 == 0)
    got = oracle.prefill_block_sparse_ref(Q, K, V, R, m, rows=[(0, 1, 200), (0, 0, 299)])
    for row, (b, h, i) in zip(got, [(0, 1, 200), (0, 0, 299)]):
        ks = [j for j in range(i + 1) if (j // 64) // 2 == i // 128 or (j // 64) % 3 == 0]
        np.testing.assert_allclose(row, oracle.parallax_row(Q[b, h, i], R[b, h, i], K[b, h, ks], V[b, h, ks]),
                                   rtol=0, atol=1e-13)
