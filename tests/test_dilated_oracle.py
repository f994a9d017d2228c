"""Pins of the dilated prefill oracle (CPU only).

Reading: query i sees keys i, i - r, i - 2r, ... (the last W of them with a
window of W keys).  What fixes it apart from the oracle's own loop: dilation 1
is the causal (windowed) prefill; a dilation of at least N leaves every row its
own key only (output v_i); each residue class mod r is an independent causal
(windowed) prefill of its own subsequence, recomputed here by slicing with the
plain prefill oracle; rows of one class ignore the inputs of every other class;
and a planted off-by-one (keys i - k r - 1) is caught.
"""
import numpy as np
import pytest

import oracle
from oracle import parallax as P


def _inputs(seed, B=1, H=2, Hkv=2, N=24, d=8):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, H, N, d)) / 2
    K = rng.standard_normal((B, Hkv, N, d)) / 2
    V = rng.standard_normal((B, Hkv, N, d))
    R = 0.25 * rng.standard_normal((B, H, N, d))
    return Q, K, V, R


@pytest.mark.parametrize("window", [None, 1, 3, 100])
def test_dilation_one_is_the_causal_or_window_prefill(window):
    Q, K, V, R = _inputs(1)
    got = oracle.prefill_dilated_ref(Q, K, V, R, 1, window)
    want = oracle.prefill_ref(Q, K, V, R, causal=True, window=window)
    assert np.allclose(got, want, rtol=0, atol=1e-13)


def test_dilation_past_the_sequence_leaves_each_row_its_own_key():
    Q, K, V, R = _inputs(2)
    got = oracle.prefill_dilated_ref(Q, K, V, R, 24)
    assert np.allclose(got, V, rtol=0, atol=1e-13)


@pytest.mark.parametrize("r,window", [(2, None), (3, None), (4, 2), (3, 5)])
def test_each_residue_class_is_a_prefill_of_its_subsequence(r, window):
    Q, K, V, R = _inputs(3, N=24)
    got = oracle.prefill_dilated_ref(Q, K, V, R, r, window)
    for rho in range(r):
        sub = slice(rho, None, r)
        want = oracle.prefill_ref(Q[:, :, sub], K[:, :, sub], V[:, :, sub], R[:, :, sub], causal=True,
                                  window=window)
        assert np.allclose(got[:, :, sub], want, rtol=0, atol=1e-13)


def test_other_classes_do_not_matter():
    Q, K, V, R = _inputs(4)
    a = oracle.prefill_dilated_ref(Q, K, V, R, 3, 4)
    K2, V2 = K.copy(), V.copy()
    K2[:, :, 1::3] += 5.0
    V2[:, :, 2::3] -= 7.0
    b = oracle.prefill_dilated_ref(Q, K2, V2, R, 3, 4)
    assert np.allclose(a[:, :, 0::3], b[:, :, 0::3], rtol=0, atol=1e-13)


def test_grouped_kv_heads():
    Q, K, V, R = _inputs(5, H=4, Hkv=2)
    got = oracle.prefill_dilated_ref(Q, K, V, R, 2)
    want = oracle.prefill_dilated_ref(Q, np.repeat(K, 2, axis=1), np.repeat(V, 2, axis=1), R, 2)
    assert np.allclose(got, want, rtol=0, atol=1e-13)


def test_planted_off_by_one_is_caught(monkeypatch):
    Q, K, V, R = _inputs(6)
    want = oracle.prefill_dilated_ref(Q, K, V, R, 3)

    def shifted(i, dilation, window=None):
        keys = np.arange(i, -1, -int(dilation), dtype=np.int64)[::-1]
        return np.maximum(keys - (keys != i), 0)  # every key but the own one moved back by one

    monkeypatch.setattr(P, "dilated_visible_keys", shifted)
    bad = oracle.prefill_dilated_ref(Q, K, V, R, 3)
    assert np.max(np.abs(bad - want)) > 1e-2
