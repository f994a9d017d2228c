"""Pins of the fp8-linear oracle (CPU only).

* e4m3 rounding: values on the e4m3 grid are kept, ties go to the even code
  (hand-worked: 1.0625 -> 1, 1.1875 -> 1.25, 232 -> 224), 448 is the largest
  value, 2^-9 the smallest subnormal;
* per-tensor scaling maps the largest magnitude to exactly 448 and keeps
  every quantised value within half an e4m3 step of the input;
* the fp8 layer with the quantiser replaced by the identity is the float64
  layer oracle (the structure is the layer's, only the linears change);
* with real quantisation the layer moves by a few percent of its RMS, as
  three-bit mantissas predict, and not by more.
"""
import numpy as np
import pytest

import oracle
from oracle import layer as olayer
from local_linear_attention_streamed_b200 import synth
from _util import small_inputs


def test_e4m3_rounding_hand_values():
    a = np.array([1.0625, 1.1875, 232.0, 240.0, 448.0, 2.0 ** -9, 2.0 ** -10, -1.0625, 0.0])
    want = np.array([1.0, 1.25, 224.0, 240.0, 448.0, 2.0 ** -9, 0.0, -1.0, 0.0])
    np.testing.assert_array_equal(oracle.e4m3(a), want)


def test_e4m3_grid_is_kept():
    # Every normal e4m3 value: (1 + m/8) 2^e, e in -6..8, m in 0..7 (but 448 = 1.75 * 2^8 is the top).
    grid = np.array([(1 + m / 8.0) * 2.0 ** e for e in range(-6, 9) for m in range(8)])
    grid = grid[grid <= 448.0]
    np.testing.assert_array_equal(oracle.e4m3(grid), grid)
    np.testing.assert_array_equal(oracle.e4m3(-grid), -grid)


def test_per_tensor_scale_and_error_bound():
    a = np.random.default_rng(1).standard_normal((64, 32)) * 3.0
    q, s = oracle.fp8_per_tensor(a)
    assert np.isclose(np.max(np.abs(q)), 448.0) and np.isclose(s, np.max(np.abs(a)) / 448.0)
    # Half a step of a 3-bit mantissa: |q s - a| <= 2^-4 |a| for normals, and
    # at most half the smallest subnormal step (2^-10 s) below them.
    err = np.abs(q * s - a)
    assert np.all(err <= np.maximum(2.0 ** -4 * np.abs(a), 2.0 ** -10 * s) + 1e-15)


def _layer_inputs(B=2, N=24, D=64, H=2, seed=5):
    _, ref = small_inputs(seed, synth.layer_specs(B, N, D), synth.F32, device="cpu")
    return ref


def test_identity_quantiser_gives_the_float64_layer():
    ref = _layer_inputs()
    H = 2
    got = oracle.layer_fp8_ref(ref["x"], ref["WQ"], ref["WK"], ref["WV"], ref["WR"], ref["WO"], H,
                               linear=lambda a, W: a @ W)
    B, N, D = ref["x"].shape
    rows = [(b, t) for b in range(B) for t in range(N)]
    want = oracle.layer_rows_ref(ref["x"], ref["WQ"], ref["WK"], ref["WV"], ref["WR"], ref["WO"], H, rows)
    np.testing.assert_allclose(got.reshape(B * N, D), want, rtol=0, atol=1e-12)


def test_fp8_layer_moves_by_a_few_percent():
    ref = _layer_inputs()
    H = 2
    got = oracle.layer_fp8_ref(ref["x"], ref["WQ"], ref["WK"], ref["WV"], ref["WR"], ref["WO"], H)
    exact = oracle.layer_fp8_ref(ref["x"], ref["WQ"], ref["WK"], ref["WV"], ref["WR"], ref["WO"], H,
                                 linear=lambda a, W: a @ W)
    rel = np.sqrt(np.mean((got - exact) ** 2) / np.mean(exact ** 2))
    assert 1e-3 < rel < 0.15, rel
