"""GPU parity of the sliding-window prefill and decode, and of the prefill fed
the exact-LLA probes, through the C ABI, against the float64 oracle.

Bars as in test_parity_gpu.py: bf16 max |g - o| / RMS(o_row) <= 2e-2 per
output row; fp32 max_e |g - o| / max(|o_e|, RMS(o)) <= 1e-5.
"""
import numpy as np
import pytest
import torch

import oracle
from local_linear_attention_streamed_b200 import synth
from _util import BF16_TOL, F32_TOL, device_inputs, rel_err_f32, rel_err_rms, small_inputs, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def plx():
    from local_linear_attention_streamed_b200 import plx as mod
    assert torch.cuda.is_available()
    return mod


@pytest.mark.parametrize("N,d,W", [(300, 128, 1), (300, 128, 37), (300, 128, 64), (300, 128, 128),
                                   (300, 128, 200), (200, 64, 5), (200, 64, 64), (200, 64, 150),
                                   (130, 128, 129), (600, 128, 256), (700, 128, 300)])
def test_prefill_window_bf16(plx, N, d, W):
    """Windows shorter than, equal to and longer than a 64-key block and a
    128-query tile, ragged N; every output row."""
    B, H = 1, 3
    dev, ref = small_inputs(700 + N + W, synth.prefill_specs(B, H, N, d), synth.BF16)
    out = plx.prefill_window(dev["Q"], dev["K"], dev["V"], dev["R"], W)
    assert plx.get_device_status() == 0
    want = oracle.prefill_ref(ref["Q"], ref["K"], ref["V"], ref["R"], window=W)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL


def test_prefill_window_covering_all_keys_is_causal(plx):
    B, H, N, d = 1, 2, 256, 128
    dev, _ = small_inputs(71, synth.prefill_specs(B, H, N, d), synth.BF16)
    a = plx.prefill_window(dev["Q"], dev["K"], dev["V"], dev["R"], N)
    b = plx.prefill(dev["Q"], dev["K"], dev["V"], dev["R"], causal=True)
    assert torch.equal(a, b)


@pytest.mark.parametrize("W", [64, 256])
@pytest.mark.parametrize("d", [64, 128])
def test_prefill_window_rescale_path(plx, d, W):
    """The causal rescale stress (keys from position 200 on scaled by 8: the
    running max jumps by far more than 2^8) with windows that straddle the
    jump, so raises and centre moves happen on rows whose first visible key
    comes after the tile's first block."""
    B, H, N = 1, 2, 520
    dev, ref = small_inputs(13, synth.prefill_specs(B, H, N, d), synth.BF16)
    dev["K"][:, :, 200:] *= 8
    ref["K"] = dev["K"].double().cpu().numpy()
    out = plx.prefill_window(dev["Q"], dev["K"], dev["V"], dev["R"], W)
    assert plx.get_device_status() == 0
    want = oracle.prefill_ref(ref["Q"], ref["K"], ref["V"], ref["R"], window=W)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL


def test_prefill_window_fp32_simt(plx):
    B, H, N, d, W = 1, 2, 150, 64, 33
    dev, ref = small_inputs(73, synth.prefill_specs(B, H, N, d, qk_dist=synth.NORMAL), synth.F32)
    out = plx.prefill_window(dev["Q"], dev["K"], dev["V"], dev["R"], W)
    want = oracle.prefill_ref(ref["Q"], ref["K"], ref["V"], ref["R"], window=W)
    assert rel_err_f32(to_f64(out), want) <= F32_TOL


@pytest.mark.parametrize("W", [1, 100, 700, 2000])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_window_bf16(plx, d, W):
    B, H, L = 5, 3, 1000
    seqlens = [1, 99, 640, 1000, 777]
    dev, ref = small_inputs(740 + W + d, synth.decode_specs(B, H, L, d), synth.BF16)
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    out = plx.decode_window(dev["q"], dev["r"], dev["K"], dev["V"], sl, W)
    torch.cuda.synchronize()
    assert plx.get_device_status() == 0
    want = oracle.decode_ref(ref["q"], ref["r"], ref["K"], ref["V"], np.asarray(seqlens), window=W)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL


@pytest.mark.parametrize("G", [2, 4, 8])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_window_grouped(plx, G, d):
    B, Hkv, L, W = 3, 2, 900, 300
    H = G * Hkv
    seqlens = [900, 250, 601]
    dev, ref = small_inputs(760 + G + d, synth.decode_gqa_specs(B, H, Hkv, L, d), synth.BF16)
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    out = plx.decode_window(dev["q"], dev["r"], dev["K"], dev["V"], sl, W)
    torch.cuda.synchronize()
    assert plx.get_device_status() == 0
    G_ = H // Hkv
    Kx = np.repeat(ref["K"], G_, axis=1)
    Vx = np.repeat(ref["V"], G_, axis=1)
    want = oracle.decode_ref(ref["q"], ref["r"], Kx, Vx, np.asarray(seqlens), window=W)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL


def test_decode_window_fp32_simt(plx):
    B, H, L, d, W = 3, 2, 300, 64, 45
    seqlens = [300, 12, 150]
    dev, ref = small_inputs(780, synth.decode_specs(B, H, L, d), synth.F32)
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    out = plx.decode_window(dev["q"], dev["r"], dev["K"], dev["V"], sl, W)
    want = oracle.decode_ref(ref["q"], ref["r"], ref["K"], ref["V"], np.asarray(seqlens), window=W)
    assert rel_err_f32(to_f64(out), want) <= F32_TOL


def test_window_rejects_bad_arguments(plx):
    x = torch.zeros((1, 1, 64, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(plx.PlxError) as e:
        plx.prefill_window(x, x, x, x, 0)
    assert e.value.code == -1
    q = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda")
    K = torch.zeros((1, 2, 64, 128), dtype=torch.bfloat16, device="cuda")
    sl = torch.tensor([64], dtype=torch.int32, device="cuda")
    with pytest.raises(plx.PlxError) as e:
        plx.decode_window(q.float(), q.float(), K.float(), K.float(), sl, 8)
    assert e.value.code == -2


def test_prefill_window_full_size_sampled(plx):
    """Sliding window of 1024 keys on the prefill workload B=8, H=16, N=4096, d=128."""
    B, H, N, d, W = 8, 16, 4096, 128, 1024
    seed = 1020
    specs = synth.prefill_specs(B, H, N, d)
    dev = device_inputs(seed, specs, synth.BF16)
    out = plx.prefill_window(dev["Q"], dev["K"], dev["V"], dev["R"], W)
    torch.cuda.synchronize()
    assert plx.get_device_status() == 0
    rng = np.random.default_rng(9)
    rows = [(0, 0, 0), (7, 15, N - 1), (3, 4, W - 1), (3, 4, W), (5, 9, 2000)]
    rows += [(int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(N))) for _ in range(10)]
    got, want = [], []
    for (b, h, i) in rows:
        row0 = (b * H + h) * N
        lo = max(0, i - W + 1)
        q = synth.host_rows_f64(seed, specs["Q"], synth.BF16, row0 + i, 1)[0]
        r = synth.host_rows_f64(seed, specs["R"], synth.BF16, row0 + i, 1)[0]
        K = synth.host_rows_f64(seed, specs["K"], synth.BF16, row0 + lo, i + 1 - lo)
        V = synth.host_rows_f64(seed, specs["V"], synth.BF16, row0 + lo, i + 1 - lo)
        want.append(oracle.parallax_row(q, r, K, V))
        got.append(to_f64(out[b, h, i]))
    assert rel_err_rms(np.stack(got), np.stack(want)) <= BF16_TOL
    assert torch.isfinite(out).all()


def test_decode_window_full_size_sampled(plx):
    """Sliding window of 1024 keys on the decode workload B=64, H=16, L=4096, d=128."""
    B, H, L, d, W = 64, 16, 4096, 128, 1024
    seed = 1021
    specs = synth.decode_specs(B, H, L, d)
    dev = device_inputs(seed, specs, synth.BF16)
    sl = torch.full((B,), L, dtype=torch.int32, device="cuda")
    out = plx.decode_window(dev["q"], dev["r"], dev["K"], dev["V"], sl, W)
    torch.cuda.synchronize()
    assert plx.get_device_status() == 0
    got, want = [], []
    for (b, h) in [(0, 0), (63, 15), (17, 3), (40, 8)]:
        bh = b * H + h
        q = synth.host_rows_f64(seed, specs["q"], synth.BF16, bh, 1)[0]
        r = synth.host_rows_f64(seed, specs["r"], synth.BF16, bh, 1)[0]
        K = synth.host_rows_f64(seed, specs["K"], synth.BF16, bh * L + L - W, W)
        V = synth.host_rows_f64(seed, specs["V"], synth.BF16, bh * L + L - W, W)
        want.append(oracle.parallax_row(q, r, K, V))
        got.append(to_f64(out[b, h]))
    assert rel_err_rms(np.stack(got), np.stack(want)) <= BF16_TOL


def _direct_fp32_row(q, rho, K, V):
    """One row of out = ((1 + T/omega) O1 - O2)/omega in plain fp32 arithmetic
    (used only to size the fp32 bar of the exact-LLA case)."""
    q, rho, K, V = (np.asarray(x, np.float32) for x in (q, rho, K, V))
    s = (K @ q) / np.float32(np.sqrt(q.shape[0]))
    w = np.exp(s - s.max())
    om = w.sum()
    t = K @ rho
    return ((1 + (w * t).sum() / om) * (w @ V) - (w * t) @ V) / om


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_with_solved_probes_is_exact_lla(plx, d):
    """Fed R = rho* (the exact-LLA solve, lambda = 1), the fp32 prefill
    evaluates Local Linear Attention itself: it matches the ridge local-linear
    intercept.  The solved probes make |t| = |rho* . k| reach ~130, so fp32
    rounding of t is amplified: the bar is four times the error of a direct
    fp32 evaluation of the same rows (fp32 rho*).  The bf16 kernel fed
    bf16(rho*) matches the oracle at those probes within the bf16 bar (the
    rounding of rho* itself moves LLA by several percent)."""
    B, H, N, lam = 1, 2, 160, 1.0
    dev, ref = small_inputs(790 + d, synth.prefill_specs(B, H, N, d), synth.F32)
    lla_out, Rs = oracle.lla_prefill_ref(ref["Q"], ref["K"], ref["V"], lam, causal=True)
    R32 = torch.from_numpy(Rs).float().cuda()
    out = plx.prefill(dev["Q"], dev["K"], dev["V"], R32, causal=True)
    direct = np.zeros_like(lla_out)
    for h in range(H):
        for i in range(N):
            direct[0, h, i] = _direct_fp32_row(ref["Q"][0, h, i], Rs[0, h, i], ref["K"][0, h, :i + 1],
                                               ref["V"][0, h, :i + 1])
    bar = max(F32_TOL, 4.0 * rel_err_f32(direct, lla_out))
    assert rel_err_f32(to_f64(out), lla_out) <= bar
    Qb, Kb, Vb = (dev[n].to(torch.bfloat16) for n in ("Q", "K", "V"))
    Rb = R32.to(torch.bfloat16)
    outb = plx.prefill(Qb, Kb, Vb, Rb, causal=True)
    want = oracle.prefill_ref(to_f64(Qb), to_f64(Kb), to_f64(Vb), to_f64(Rb), causal=True)
    assert rel_err_rms(to_f64(outb), want) <= BF16_TOL
