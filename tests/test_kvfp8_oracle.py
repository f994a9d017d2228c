"""Pins of the fp8 (e4m3) KV-cache oracle (CPU only).

The quantiser reading (oracle/kvfp8.py): each cache row gets its own scale
s = max|x| / 448 and codes e4m3(x / s), divisions in float32, round to
nearest with ties to even.  What fixes it independently of the oracle's own
code: the e4m3 format itself (1 sign, 4 exponent bits with bias 7, 3 mantissa
bits; subnormals m * 2^-9; largest finite 448; encoding sign<<7 | E<<3 | m),
which the tests enumerate from that definition; hand-worked ties; the
half-step error bound; the row maximum landing on 448; and the identity
case, a cache already on the grid, where the fp8 decode must equal the plain
decode.  Planted mistakes (truncation, a 240 maximum, a scale left out) are
caught.
"""
import numpy as np
import pytest

import oracle
from oracle import kvfp8


def _grid():
    """Every non-negative finite e4m3 value with its encoding, from the format's definition."""
    vals, bits = [], []
    for E in range(16):
        for m in range(8):
            if E == 15 and m == 7:
                continue  # the NaN encoding
            vals.append(m * 2.0 ** -9 if E == 0 else 2.0 ** (E - 7) * (1 + m / 8))
            bits.append((E << 3) | m)
    return np.array(vals), np.array(bits, dtype=np.uint8)


def _spacing(y):
    """Distance between adjacent e4m3 values around |y| (<= 448)."""
    a = np.abs(y)
    E = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return np.where(a < 2.0 ** -6, 2.0 ** -9, 2.0 ** (E - 3))


def _check_pins(quantize):
    """Runs every pin against a quantiser; returns the first failure (or None)."""
    vals, bits = _grid()
    # Hand-worked ties at scale 1 (the row holds 448): 1.0625 lies midway
    # between 1 and 1.125 (even mantissa: 1), 1.1875 between 1.125 and 1.25
    # (even: 1.25), 232 between 224 and 240 (even: 224), 1.5 * 2^-9 between the
    # subnormals 2^-9 and 2^-8 (even: 2^-8).
    x = np.array([[448.0, 1.0625, 1.1875, 232.0, 1.5 * 2.0 ** -9, -1.0625, 0.0, 2.0 ** -9]])
    c, s = quantize(x)
    want = np.array([[448.0, 1.0, 1.25, 224.0, 2.0 ** -8, -1.0, 0.0, 2.0 ** -9]])
    if not (s[0] == 1.0 and np.array_equal(oracle.kv_dequantize_fp8_ref(c, s), want)):
        return "hand ties"
    # The whole grid, both signs, scaled by powers of two: kept exactly, with
    # the encodings the format defines.
    for k in (-12, 0, 5):
        row = np.concatenate([vals, -vals[1:]]) * 2.0 ** k
        c, s = quantize(row[None])
        if s[0] != 2.0 ** k or not np.array_equal(oracle.kv_dequantize_fp8_ref(c, s)[0], row):
            return "grid kept"
        if not np.array_equal(c[0], np.concatenate([bits, bits[1:] | 0x80])):
            return "encodings"
    # Random rows: within half a step of the e4m3 grid at x / s (plus the
    # float32 division's rounding); the row maximum lands on 448.
    rng = np.random.default_rng(7)
    X = rng.standard_normal((64, 128)) * np.exp(rng.uniform(-20, 20, size=(64, 1)))
    X = X.astype(np.float32).astype(np.float64)
    c, s = quantize(X)
    y = X / s[:, None]
    err = np.abs(oracle.kv_dequantize_fp8_ref(c, s) - X)
    if not np.all(err <= (0.5 * _spacing(y) * (1 + 1e-6) + np.abs(y) * 2.0 ** -22) * s[:, None]):
        return "half step"
    if not np.all(np.max(np.abs(kvfp8.e4m3_value(c)), axis=1) == 448.0):
        return "max on 448"
    # Sign symmetry and the zero row.
    c2, s2 = quantize(-X)
    if not (np.array_equal(s2, s) and np.array_equal(kvfp8.e4m3_value(c2), -kvfp8.e4m3_value(c))):
        return "sign"
    c0, s0 = quantize(np.zeros((1, 128)))
    if not (s0[0] == 0 and np.all(c0 == 0)):
        return "zero row"
    return None


def test_quantiser_pins():
    assert _check_pins(oracle.kv_quantize_fp8_ref) is None


def test_planted_quantiser_mistakes_are_caught(monkeypatch):
    def truncating(X):
        x32 = np.asarray(X, dtype=np.float64).astype(np.float32)
        s = (np.max(np.abs(x32), axis=-1) / np.float32(448)).astype(np.float32)
        y = np.where(s[..., None] > 0, x32 / np.where(s > 0, s, 1)[..., None], 0).astype(np.float64)
        vals, _ = _grid()
        a = np.abs(y)
        idx = np.searchsorted(vals, a, side="right") - 1  # round toward zero
        return kvfp8.e4m3_bits(np.sign(y) * vals[idx]), s

    assert _check_pins(truncating) == "hand ties"
    with monkeypatch.context() as m:
        m.setattr(kvfp8, "E4M3_MAX", 240.0)  # the e4m3fnuz maximum
        assert _check_pins(kvfp8.kv_quantize_fp8_ref) is not None

    def unscaled(X):
        c, s = oracle.kv_quantize_fp8_ref(X)
        return c, np.ones_like(s)

    assert _check_pins(unscaled) is not None


def test_identity_cache_gives_the_plain_decode():
    """A cache whose rows are already e4m3 values times a power of two is kept
    exactly, so the fp8 decode equals the plain grouped decode."""
    rng = np.random.default_rng(3)
    vals, _ = _grid()
    B, H, Hkv, L, d = 2, 4, 2, 40, 16
    K = rng.choice(np.concatenate([vals, -vals]), size=(B, Hkv, L, d))
    V = rng.choice(np.concatenate([vals, -vals]), size=(B, Hkv, L, d))
    K[..., 0] = 448.0
    V[..., 3] = -448.0
    K *= 2.0 ** rng.integers(-10, 4, size=(B, Hkv, L, 1))
    V *= 2.0 ** rng.integers(-10, 4, size=(B, Hkv, L, 1))
    q = rng.standard_normal((B, H, d)) / 40
    r = rng.standard_normal((B, H, d)) * 0.01
    sl = np.array([L, 7])
    Kc, Ks = oracle.kv_quantize_fp8_ref(K)
    Vc, Vs = oracle.kv_quantize_fp8_ref(V)
    got = oracle.decode_fp8kv_ref(q, r, Kc, Ks, Vc, Vs, sl)
    want = oracle.decode_gqa_ref(q, r, K, V, sl)
    assert np.max(np.abs(got - want)) <= 1e-12 * np.max(np.abs(want))


def test_decode_over_quantised_cache_is_close_to_the_bf16_decode():
    """Sanity of scale handling end to end: on the decode workload's
    distributions the fp8 cache moves outputs by a few percent of their RMS
    (e4m3 keeps 4 significant bits), not by O(1)."""
    rng = np.random.default_rng(11)
    B, H, Hkv, L, d = 2, 4, 4, 300, 128
    K = rng.standard_normal((B, Hkv, L, d))
    K /= np.sqrt(np.mean(K * K, axis=-1, keepdims=True))
    V = rng.standard_normal((B, Hkv, L, d))
    q = rng.standard_normal((B, H, d))
    q /= np.sqrt(np.mean(q * q, axis=-1, keepdims=True))
    r = 0.25 * rng.standard_normal((B, H, d))
    sl = np.array([300, 150])
    Kc, Ks = oracle.kv_quantize_fp8_ref(K)
    Vc, Vs = oracle.kv_quantize_fp8_ref(V)
    got = oracle.decode_fp8kv_ref(q, r, Kc, Ks, Vc, Vs, sl)
    want = oracle.decode_gqa_ref(q, r, K, V, sl)
    rel = np.sqrt(np.mean((got - want) ** 2) / np.mean(want * want))
    assert 1e-3 < rel < 0.15


def test_three_e4m3_terms_hold_a_scaled_bf16_row():
    """The e4m3-cache decode feeds q and rho to e4m3 score MMAs as three e4m3
    terms per element (hi, then the rounding of what is left, twice), after
    scaling the row by the power of two that puts its largest element in
    [2^7, 2^8).  With round-to-nearest e4m3 (subnormals included) the three
    terms give back every bf16 element to within 2^-17 of the row's largest,
    so the three score columns add up to the score of the unrounded operand;
    two terms do not (errors near 2^-9 of an element)."""
    import torch
    from oracle.layer import e4m3

    rng = np.random.default_rng(5)
    rows = rng.standard_normal((64, 128)) * 2.0 ** rng.uniform(-12, 0, (64, 128))
    rows[0, 3] *= 2.0 ** 10                      # one element far above the rest
    rows[1] = 0.0
    rows[1, 7] = -3.0                            # a single non-zero element
    x = torch.from_numpy(rows).to(torch.bfloat16).double().numpy()
    worst3, worst2 = 0.0, 0.0
    for row in x:
        m = np.max(np.abs(row))
        if m == 0:
            continue
        e = int(np.floor(np.log2(m))) - 7
        y = np.ldexp(row, -e)
        assert 2.0 ** 7 <= np.max(np.abs(y)) < 2.0 ** 8
        t1 = e4m3(y)
        t2 = e4m3(y - t1)
        t3 = e4m3(y - t1 - t2)
        worst3 = max(worst3, np.max(np.abs(y - (t1 + t2 + t3))) / np.max(np.abs(y)))
        worst2 = max(worst2, np.max(np.abs((y - (t1 + t2)) / np.where(y == 0, 1, y))))
    assert worst3 <= 2.0 ** -17
    assert worst2 > 2.0 ** -10


def test_e4m3_to_bf16_bit_moves_are_exact():
    """The e4m3-cache decode converts value codes to bf16 with integer bit
    moves: the code in the high byte of a 16-bit lane, its sign kept and its 7
    exponent and mantissa bits shifted right by 4, is a bf16 whose value is
    the code's times 2^-120 (exponent bias 7 against 127; the e4m3 subnormals
    land on bf16 subnormals), and one multiply by 2^120 restores it.  Checked
    for every finite code against the format's own decoding."""
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint32)
    lane = codes << 8
    bf16_bits = (lane & 0x8000) | ((lane & 0x7F00) >> 4)
    as_f32 = (bf16_bits << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    want = oracle.e4m3_value(codes.astype(np.uint8))
    assert np.array_equal(as_f32 * 2.0 ** 120, want)
    assert np.array_equal(np.sign(as_f32), np.sign(want))
