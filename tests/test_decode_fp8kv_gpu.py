"""GPU parity of the e4m3 KV cache: the quantiser (plx_kv_quantize_fp8) bit for
bit against the oracle's quantiser, and the decode over the quantised cache
(plx_decode_fp8kv) against the float64 oracle decode over the cache values.

The oracle quantises the same bf16 rows itself (oracle.kv_quantize_fp8_ref);
nothing the GPU writes is fed to it.  Codes are integer results: bit-exact.
Decode bar: max |g - o| / RMS(o) <= 2e-2 per output vector (bf16 outputs).
"""
import numpy as np
import pytest
import torch

import oracle
from local_linear_attention_streamed_b200 import synth
from _util import BF16_TOL, device_inputs, rel_err_rms, small_inputs, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def plx():
    from local_linear_attention_streamed_b200 import plx as mod
    assert torch.cuda.is_available()
    return mod


def _bf16(a):
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.cuda(), t.double().numpy()


@pytest.mark.parametrize("d", [64, 128])
def test_quantiser_codes_and_scales_are_bit_exact(plx, d):
    rng = np.random.default_rng(d)
    rows = [rng.standard_normal(d) * np.exp(rng.uniform(-30, 30)) for _ in range(300)]
    rows.append(np.zeros(d))                                  # zero row
    rows.append(np.full(d, -3.0))                             # constant row
    grid = np.array([448.0, 1.0625, 1.1875, 232.0, 1.5 * 2 ** -9, 2 ** -9, -1.0625, 0.0])
    rows.append(np.resize(grid, d))                           # hand ties at scale 1
    rows.append(np.resize(grid, d) * 2.0 ** -20)              # the same ties at scale 2^-20
    X, Xr = _bf16(np.stack(rows))
    codes, scales = plx.kv_quantize_fp8(X)
    torch.cuda.synchronize()
    want_c, want_s = oracle.kv_quantize_fp8_ref(Xr)
    assert np.array_equal(codes.cpu().numpy(), want_c)
    assert np.array_equal(scales.cpu().numpy(), want_s)


def _fp8_case(plx, dev_K, dev_V, ref_K, ref_V):
    Kc, Ks = plx.kv_quantize_fp8(dev_K)
    Vc, Vs = plx.kv_quantize_fp8(dev_V)
    oKc, oKs = oracle.kv_quantize_fp8_ref(ref_K)
    oVc, oVs = oracle.kv_quantize_fp8_ref(ref_V)
    torch.cuda.synchronize()
    assert np.array_equal(Kc.cpu().numpy(), oKc) and np.array_equal(Vc.cpu().numpy(), oVc)
    assert np.array_equal(Ks.cpu().numpy(), oKs) and np.array_equal(Vs.cpu().numpy(), oVs)
    return (Kc, Ks, Vc, Vs), (oKc, oKs, oVc, oVs)


@pytest.mark.parametrize("G,Hkv", [(1, 3), (2, 2), (4, 2), (8, 1)])
def test_fp8kv_small_ragged(plx, G, Hkv):
    """Every output; lengths at the 128-key block edges and a ragged tail."""
    B, L, d = 6, 600, 128
    H = G * Hkv
    specs = synth.decode_gqa_specs(B, H, Hkv, L, d)
    dev, ref = small_inputs(80 + G, specs, synth.BF16)
    gpu, orc = _fp8_case(plx, dev["K"], dev["V"], ref["K"], ref["V"])
    sl = np.array([1, 127, 128, 129, 600, 300], dtype=np.int32)
    out = plx.decode_fp8kv(dev["q"], dev["r"], *gpu, torch.from_numpy(sl).cuda())
    assert plx.get_device_status() == 0
    want = oracle.decode_fp8kv_ref(ref["q"], ref["r"], *orc, sl)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL


@pytest.mark.parametrize("G", [1, 4, 8])
def test_fp8kv_split_keys_repeatable(plx, G):
    """Few (b, KV head) pairs over long caches: keys cut into chunks merged in-kernel."""
    B, Hkv, L, d = 1, 2, 8192, 128
    H = G * Hkv
    assert plx.decode_fp8kv_workspace_bytes(B, H, Hkv, L, d) > 0
    specs = synth.decode_gqa_specs(B, H, Hkv, L, d)
    dev, ref = small_inputs(90 + G, specs, synth.BF16)
    gpu, orc = _fp8_case(plx, dev["K"], dev["V"], ref["K"], ref["V"])
    sl = np.array([L - 37], dtype=np.int32)
    out = plx.decode_fp8kv(dev["q"], dev["r"], *gpu, torch.from_numpy(sl).cuda())
    assert plx.get_device_status() == 0
    want = oracle.decode_fp8kv_ref(ref["q"], ref["r"], *orc, sl)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL
    out2 = plx.decode_fp8kv(dev["q"], dev["r"], *gpu, torch.from_numpy(sl).cuda())
    assert torch.equal(out, out2)
    ws = torch.zeros(plx.decode_fp8kv_workspace_bytes(B, H, Hkv, L, d), dtype=torch.uint8, device="cuda")
    out3 = plx.decode_fp8kv(dev["q"], dev["r"], *gpu, torch.from_numpy(sl).cuda(), workspace=ws)
    assert torch.equal(out, out3)


def test_fp8kv_garbage_past_the_lengths_does_not_leak(plx):
    """NaN codes (0x7f) and NaN scales past every sequence's length."""
    B, H, Hkv, L, d = 4, 8, 2, 700, 128
    specs = synth.decode_gqa_specs(B, H, Hkv, L, d)
    dev, ref = small_inputs(97, specs, synth.BF16)
    (Kc, Ks, Vc, Vs), orc = _fp8_case(plx, dev["K"], dev["V"], ref["K"], ref["V"])
    sl = np.array([700, 1, 200, 333], dtype=np.int32)
    for b in range(B):
        for t in (Kc, Vc):
            t[b, :, sl[b]:] = 0x7F
        for t in (Ks, Vs):
            t[b, :, sl[b]:] = float("nan")
    out = plx.decode_fp8kv(dev["q"], dev["r"], Kc, Ks, Vc, Vs, torch.from_numpy(sl).cuda())
    assert plx.get_device_status() == 0
    assert torch.isfinite(out).all()
    want = oracle.decode_fp8kv_ref(ref["q"], ref["r"], *orc, sl)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL


def test_fp8kv_subnormal_codes(plx):
    """Rows whose first element is 10^5 times the rest: after scaling by
    max / 448 the other elements fall in e4m3's subnormal range (2^-9 .. 2^-6)
    or round to zero, in K and in V.  Dims 1..127 of the output are then made
    of subnormal-coded values only, and are compared on their own RMS."""
    B, H, Hkv, L, d = 2, 4, 2, 400, 128
    rng = np.random.default_rng(96)
    K = rng.standard_normal((B, Hkv, L, d))
    V = rng.standard_normal((B, Hkv, L, d))
    for X in (K, V):
        X[..., 0] = 1e5 * np.where(rng.random((B, Hkv, L)) < 0.5, 1.0, -1.0)
    K /= 1e4
    q = rng.standard_normal((B, H, d))
    r = 0.25 * rng.standard_normal((B, H, d))
    (Kd, Kr), (Vd, Vr), (qd, qr), (rd, rr) = _bf16(K), _bf16(V), _bf16(q), _bf16(r)
    gpu, orc = _fp8_case(plx, Kd, Vd, Kr, Vr)
    for codes in (orc[0], orc[2]):
        sub = (codes[..., 1:] & 0x78) == 0
        nonzero = (codes[..., 1:] & 0x7F) != 0
        assert np.mean(sub & nonzero) > 0.4  # subnormal codes, not zeros
    sl = np.array([400, 257], dtype=np.int32)
    out = plx.decode_fp8kv(qd, rd, *gpu, torch.from_numpy(sl).cuda())
    assert plx.get_device_status() == 0
    want = oracle.decode_fp8kv_ref(qr, rr, *orc, sl)
    got = to_f64(out)
    # Dim 0 dominates each output vector, so bf16 output rounding alone moves it
    # by up to 2^-9 sqrt(128) = 2.2 % of the vector's RMS: it is held to its own
    # value (rounding 2^-9 plus accumulation), the subnormal-coded dims to the bar.
    assert np.all(np.abs(got[..., 0] - want[..., 0]) <= 2.0 ** -7 * np.abs(want[..., 0]))
    assert rel_err_rms(got[..., 1:], want[..., 1:]) <= BF16_TOL


@pytest.mark.parametrize("key_scale", [1.0, 3.0])
def test_fp8kv_true_normal(plx, key_scale):
    """Unbounded normal draws (q, k RMS rows, keys optionally x 3; v ~ N(0, 1); rho ~ N(0, 0.25^2))."""
    B, H, Hkv, L, d = 4, 8, 4, 1500, 128
    rng = np.random.default_rng(98)
    def rms(x):
        return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True))
    q, qr = _bf16(rms(rng.standard_normal((B, H, d))))
    r, rr = _bf16(0.25 * rng.standard_normal((B, H, d)))
    K, Kr = _bf16(key_scale * rms(rng.standard_normal((B, Hkv, L, d))))
    V, Vr = _bf16(rng.standard_normal((B, Hkv, L, d)))
    gpu, orc = _fp8_case(plx, K, V, Kr, Vr)
    sl = np.array([1500, 2, 777, 1024], dtype=np.int32)
    out = plx.decode_fp8kv(q, r, *gpu, torch.from_numpy(sl).cuda())
    assert plx.get_device_status() == 0
    want = oracle.decode_fp8kv_ref(qr, rr, *orc, sl)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_fp8kv_wide_range_queries(plx, G):
    """q and rho rows whose elements span many binades (|x| ~ 2^U(-12, 0)), and
    rows with one element 2^10 times the rest: the score operand must keep the
    small elements too.  Keys x 3 make the softmax sharp, so score errors show."""
    B, Hkv, L, d = 3, 2, 700, 128
    H = G * Hkv
    rng = np.random.default_rng(140 + G)
    def rms(x):
        return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True))
    def wide(shape):
        return rng.standard_normal(shape) * 2.0 ** rng.uniform(-12, 0, shape)
    qh = rms(wide((B, H, d)))
    rh = 0.25 * rms(wide((B, H, d)))
    qh[0, :, 5] *= 2.0 ** 10
    rh[1, :, 77] *= 2.0 ** 10
    q, qr = _bf16(qh)
    r, rr = _bf16(rh)
    K, Kr = _bf16(3.0 * rms(rng.standard_normal((B, Hkv, L, d))))
    V, Vr = _bf16(rng.standard_normal((B, Hkv, L, d)))
    gpu, orc = _fp8_case(plx, K, V, Kr, Vr)
    sl = np.array([700, 129, 512], dtype=np.int32)
    out = plx.decode_fp8kv(q, r, *gpu, torch.from_numpy(sl).cuda())
    assert plx.get_device_status() == 0
    want = oracle.decode_fp8kv_ref(qr, rr, *orc, sl)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL


@pytest.mark.parametrize("Hkv", [16, 4])
def test_fp8kv_decode_workload_sampled(plx, Hkv):
    """The decode workload's shape (B=64, H=16, L=4096, d=128, all lengths 4096)
    over an e4m3 cache, ungrouped and in groups of 4: sampled (b, h) against
    the oracle, which quantises the generator's host copy of exactly their rows."""
    B, H, L, d = 64, 16, 4096, 128
    G = H // Hkv
    seed = 1002
    specs = synth.decode_gqa_specs(B, H, Hkv, L, d)
    dev = device_inputs(seed, specs, synth.BF16)
    Kc, Ks = plx.kv_quantize_fp8(dev["K"])
    Vc, Vs = plx.kv_quantize_fp8(dev["V"])
    sl = torch.full((B,), L, dtype=torch.int32, device="cuda")
    out = plx.decode_fp8kv(dev["q"], dev["r"], Kc, Ks, Vc, Vs, sl)
    assert plx.get_device_status() == 0
    rng = np.random.default_rng(12 + Hkv)
    units = [(0, 0), (B - 1, H - 1)] + [(int(rng.integers(B)), int(rng.integers(H))) for _ in range(10)]
    got, want = [], []
    for (b, h) in units:
        kv = h // G
        r0 = (b * Hkv + kv) * L
        K = synth.host_rows_f64(seed, specs["K"], synth.BF16, r0, L)
        V = synth.host_rows_f64(seed, specs["V"], synth.BF16, r0, L)
        kc, ks = oracle.kv_quantize_fp8_ref(K)
        vc, vs = oracle.kv_quantize_fp8_ref(V)
        assert np.array_equal(Kc[b, kv].cpu().numpy(), kc) and np.array_equal(Vs[b, kv].cpu().numpy(), vs)
        qv = synth.host_rows_f64(seed, specs["q"], synth.BF16, b * H + h, 1)[0]
        rv = synth.host_rows_f64(seed, specs["r"], synth.BF16, b * H + h, 1)[0]
        want.append(oracle.parallax_row(qv, rv, oracle.kv_dequantize_fp8_ref(kc, ks),
                                        oracle.kv_dequantize_fp8_ref(vc, vs)))
        got.append(out[b, h].double().cpu().numpy())
    assert rel_err_rms(np.stack(got), np.stack(want)) <= BF16_TOL
    assert torch.isfinite(out).all()
    del dev, Kc, Vc
    torch.cuda.empty_cache()


def test_fp8kv_errors(plx):
    B, H, Hkv, L = 2, 4, 2, 256
    q = torch.zeros(B, H, 64, dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(B, Hkv, L, 64, dtype=torch.uint8, device="cuda")
    s = torch.ones(B, Hkv, L, dtype=torch.float32, device="cuda")
    sl = torch.full((B,), L, dtype=torch.int32, device="cuda")
    with pytest.raises(plx.PlxError) as e:
        plx.decode_fp8kv(q, q, c, s, c, s, sl)
    assert e.value.code == -2  # d = 64
    dev, ref = small_inputs(99, synth.decode_gqa_specs(B, H, Hkv, L, 128), synth.BF16)
    Kc, Ks = plx.kv_quantize_fp8(dev["K"])
    Vc, Vs = plx.kv_quantize_fp8(dev["V"])
    bad = torch.tensor([0, L + 1], dtype=torch.int32, device="cuda")
    out = plx.decode_fp8kv(dev["q"], dev["r"], Kc, Ks, Vc, Vs, bad)
    assert plx.get_device_status() == -6
    assert torch.all(out == 0)
