"""GPU parity of the dilated prefill (plx_prefill_dilated) against the float64
oracle: query i sees keys i, i - r, i - 2r, ... (the last W of them with a
window).  bf16 bar: max |g - o| / RMS(o) <= 2e-2 per output vector, over every
output of small cases (several tiles per residue class, ragged class tails)
and sampled rows of a large one.
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


def _specs(B, H, Hkv, N, d):
    specs = synth.prefill_specs(B, H, N, d)
    specs["K"] = synth.TensorSpec(synth.TID_K, (B, Hkv, N, d), specs["K"].dist, specs["K"].sigma)
    specs["V"] = synth.TensorSpec(synth.TID_V, (B, Hkv, N, d), specs["V"].dist, specs["V"].sigma)
    return specs


@pytest.mark.parametrize("N,r,window", [(256, 2, 0), (300, 3, 0), (384, 4, 0), (600, 2, 0), (384, 3, 5),
                                        (600, 4, 40), (520, 2, 200)])
@pytest.mark.parametrize("d", [64, 128])
def test_dilated_matches_oracle(plx, N, r, window, d):
    B, H, Hkv = 2, 4, 2
    dev, ref = small_inputs(1300 + N + r + d, _specs(B, H, Hkv, N, d), synth.BF16)
    out = plx.prefill_dilated(dev["Q"], dev["K"], dev["V"], dev["R"], r, window)
    assert plx.get_device_status() == 0
    want = oracle.prefill_dilated_ref(ref["Q"], ref["K"], ref["V"], ref["R"], r, window or None)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL


@pytest.mark.parametrize("window", [0, 100])
def test_dilation_one_is_the_grouped_prefill(plx, window):
    B, H, Hkv, N, d = 1, 4, 2, 300, 128
    dev, _ = small_inputs(1350, _specs(B, H, Hkv, N, d), synth.BF16)
    a = plx.prefill_dilated(dev["Q"], dev["K"], dev["V"], dev["R"], 1, window)
    b = plx.prefill_gqa(dev["Q"], dev["K"], dev["V"], dev["R"], causal=True, window=window or None)
    assert torch.equal(a, b)


def test_dilated_large_sampled(plx):
    """B=2, H=8, N=4096, d=128, dilation 8 (512-row classes), sampled rows of every class."""
    B, H, N, d, r = 2, 8, 4096, 128, 8
    seed = 1360
    specs = _specs(B, H, H, N, d)
    dev = device_inputs(seed, specs, synth.BF16)
    out = plx.prefill_dilated(dev["Q"], dev["K"], dev["V"], dev["R"], r, 0)
    assert plx.get_device_status() == 0
    rng = np.random.default_rng(7)
    rows = [(0, 0, 0), (0, 0, 7), (1, 7, N - 1), (1, 3, N - 8)] + \
        [(int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(N))) for _ in range(12)]
    got, want = [], []
    for (b, h, i) in rows:
        base = (b * H + h) * N
        Kh = synth.host_rows_f64(seed, specs["K"], synth.BF16, base, N)
        Vh = synth.host_rows_f64(seed, specs["V"], synth.BF16, base, N)
        q = synth.host_rows_f64(seed, specs["Q"], synth.BF16, base + i, 1)[0]
        rr = synth.host_rows_f64(seed, specs["R"], synth.BF16, base + i, 1)[0]
        ks = np.arange(i, -1, -r)[::-1]
        want.append(oracle.parallax_row(q, rr, Kh[ks], Vh[ks]))
        got.append(out[b, h, i].double().cpu().numpy())
    assert rel_err_rms(np.stack(got), np.stack(want)) <= BF16_TOL
    assert torch.isfinite(out).all()


def test_dilated_rejects_ragged_classes(plx):
    x = torch.zeros(1, 2, 300, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(plx.PlxError) as e:
        plx.prefill_dilated(x, x, x, x, 7, 0)  # 300 is not a multiple of 7
    assert e.value.code == -2
