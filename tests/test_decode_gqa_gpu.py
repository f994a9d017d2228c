"""GPU parity of the grouped-KV decode (plx_decode_gqa) against the float64 oracle.

Query head h reads KV head h // G.  Small cases compare every output; the
full-size case samples (b, h) and recomputes them from the generator's host
copy of exactly the rows each needs.  bf16 bar: max |g - o| / RMS(o) <= 2e-2
per output vector.
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


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G,Hkv", [(2, 3), (4, 2), (8, 1), (8, 2)])
def test_gqa_small_ragged(plx, d, G, Hkv):
    """Every output; lengths 1, 15, 64, 65, 200 and L (ragged tails of 64-key blocks)."""
    B, L = 6, 256
    H = G * Hkv
    specs = synth.decode_gqa_specs(B, H, Hkv, L, d)
    dev, ref = small_inputs(40 + G + d, specs, synth.BF16)
    sl_host = np.array([1, 15, 64, 65, 200, L], dtype=np.int32)
    out = plx.decode_gqa(dev["q"], dev["r"], dev["K"], dev["V"], torch.from_numpy(sl_host).cuda())
    assert plx.get_device_status() == 0
    want = oracle.decode_gqa_ref(ref["q"], ref["r"], ref["K"], ref["V"], sl_host)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [2, 4, 8])
def test_gqa_split_keys(plx, G, d):
    """Few (b, KV head) pairs and long contexts: keys split into chunks merged
    in-kernel (at d = 64 the two KV heads form one unit of the tensor-core kernel)."""
    B, Hkv, L = 1, 2, 8192
    H = G * Hkv
    assert plx.lib.plx_decode_num_splits(B, Hkv, L, d) > 1
    specs = synth.decode_gqa_specs(B, H, Hkv, L, d)
    dev, ref = small_inputs(60 + G + d, specs, synth.BF16)
    sl_host = np.array([L - 37], dtype=np.int32)
    out = plx.decode_gqa(dev["q"], dev["r"], dev["K"], dev["V"], torch.from_numpy(sl_host).cuda())
    assert plx.get_device_status() == 0
    want = oracle.decode_gqa_ref(ref["q"], ref["r"], ref["K"], ref["V"], sl_host)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL
    # The same call again (counters were left at zero) gives the same bits.
    out2 = plx.decode_gqa(dev["q"], dev["r"], dev["K"], dev["V"], torch.from_numpy(sl_host).cuda())
    assert torch.equal(out, out2)


def test_gqa_matches_ungrouped_decode_on_repeated_heads(plx):
    """Grouped decode equals the ungrouped kernel run on the KV heads repeated G times."""
    B, Hkv, G, L, d = 4, 2, 4, 1024, 128
    H = G * Hkv
    specs = synth.decode_gqa_specs(B, H, Hkv, L, d)
    dev, ref = small_inputs(71, specs, synth.BF16)
    sl = torch.tensor([1024, 700, 64, 333], dtype=torch.int32, device="cuda")
    got = plx.decode_gqa(dev["q"], dev["r"], dev["K"], dev["V"], sl)
    Kr = dev["K"].repeat_interleave(G, dim=1).contiguous()
    Vr = dev["V"].repeat_interleave(G, dim=1).contiguous()
    mha = plx.decode(dev["q"], dev["r"], Kr, Vr, sl)
    assert plx.get_device_status() == 0
    want = oracle.decode_gqa_ref(ref["q"], ref["r"], ref["K"], ref["V"], sl.cpu().numpy())
    assert rel_err_rms(to_f64(got), want) <= BF16_TOL
    assert rel_err_rms(to_f64(got), to_f64(mha)) <= BF16_TOL


def test_gqa_group_of_one_is_the_ungrouped_decode(plx):
    B, H, L, d = 3, 4, 512, 64
    specs = synth.decode_gqa_specs(B, H, H, L, d)
    dev, _ = small_inputs(72, specs, synth.BF16)
    sl = torch.tensor([512, 100, 7], dtype=torch.int32, device="cuda")
    a = plx.decode_gqa(dev["q"], dev["r"], dev["K"], dev["V"], sl)
    b = plx.decode(dev["q"], dev["r"], dev["K"], dev["V"], sl)
    assert torch.equal(a, b)


@pytest.mark.parametrize("d", [64, 128])
def test_gqa_cache_past_seqlen_never_leaks(plx, d):
    """NaN in the cache past each sequence's length must not reach the outputs."""
    B, Hkv, G, L = 3, 2, 8, 320
    H = G * Hkv
    specs = synth.decode_gqa_specs(B, H, Hkv, L, d)
    dev, ref = small_inputs(73, specs, synth.BF16)
    sl_host = np.array([70, 129, 320], dtype=np.int32)
    for b in range(B):
        dev["K"][b, :, sl_host[b]:] = float("nan")
        dev["V"][b, :, sl_host[b]:] = float("nan")
    out = plx.decode_gqa(dev["q"], dev["r"], dev["K"], dev["V"], torch.from_numpy(sl_host).cuda())
    assert plx.get_device_status() == 0
    assert torch.isfinite(out).all()
    want = oracle.decode_gqa_ref(ref["q"], ref["r"], ref["K"], ref["V"], sl_host)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL


@pytest.mark.parametrize("d", [64, 128])
def test_gqa_bad_seqlen_reports_and_zeroes(plx, d):
    B, Hkv, G, L = 3, 2, 4, 256
    H = G * Hkv
    specs = synth.decode_gqa_specs(B, H, Hkv, L, d)
    dev, ref = small_inputs(74, specs, synth.BF16)
    sl = torch.tensor([256, 0, 257], dtype=torch.int32, device="cuda")
    out = plx.decode_gqa(dev["q"], dev["r"], dev["K"], dev["V"], sl)
    assert plx.get_device_status() == -6
    assert plx.get_device_status() == 0
    o = to_f64(out)
    assert np.all(o[1] == 0) and np.all(o[2] == 0)
    want = oracle.decode_gqa_ref(ref["q"], ref["r"], ref["K"], ref["V"], np.array([256, 1, 1]),
                                 units=[(0, h) for h in range(H)])
    assert rel_err_rms(o[0], want) <= BF16_TOL


@pytest.mark.parametrize("H,Hkv", [(32, 8), (64, 8)])
def test_gqa_full_size_sampled(plx, H, Hkv):
    """Grouped decode at full size (B=64, L=4096, d=128, ragged lengths): groups of 4
    (the bench's grouped workload) and of 8."""
    B, L, d = 64, 4096, 128
    G = H // Hkv
    seed = 1005
    specs = synth.decode_gqa_specs(B, H, Hkv, L, d)
    dev = device_inputs(seed, specs, synth.BF16)
    sl_host = synth.seqlens(seed, B, L, ragged=True)
    out = plx.decode_gqa(dev["q"], dev["r"], dev["K"], dev["V"], torch.from_numpy(sl_host).cuda())
    assert plx.get_device_status() == 0
    rng = np.random.default_rng(5)
    units = [(0, 0), (B - 1, H - 1)] + [(int(rng.integers(B)), int(rng.integers(H))) for _ in range(10)]
    got, want = [], []
    for (b, h) in units:
        n = int(sl_host[b])
        r0 = (b * Hkv + h // G) * L
        K = synth.host_rows_f64(seed, specs["K"], synth.BF16, r0, n)
        V = synth.host_rows_f64(seed, specs["V"], synth.BF16, r0, n)
        q = synth.host_rows_f64(seed, specs["q"], synth.BF16, b * H + h, 1)[0]
        r = synth.host_rows_f64(seed, specs["r"], synth.BF16, b * H + h, 1)[0]
        want.append(oracle.parallax_row(q, r, K, V))
        got.append(out[b, h].double().cpu().numpy())
    assert rel_err_rms(np.stack(got), np.stack(want)) <= BF16_TOL
    assert torch.isfinite(out).all()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [2, 4, 8])
def test_gqa_rising_scores_rescale(plx, G, d):
    """Scores that grow along the sequence (K rows scaled by 1 + 20 j / L): the
    running max rises block after block, so the accumulated products are
    rescaled many times (in the d = 128 kernel, in TMEM) before the last one;
    one (b, KV head) with a single chunk and one split into chunks."""
    B, Hkv, L = 2, 2, 2048
    H = G * Hkv
    specs = synth.decode_gqa_specs(B, H, Hkv, L, d)
    dev, ref = small_inputs(90 + G + d, specs, synth.BF16)
    ramp = 1.0 + 20.0 * np.arange(L) / L
    Kh = (ref["K"] * ramp[None, None, :, None])
    dev["K"] = torch.from_numpy(Kh).to(torch.bfloat16).cuda()
    ref["K"] = dev["K"].to(torch.float64).cpu().numpy()
    sl_host = np.array([L, 1500], dtype=np.int32)
    out = plx.decode_gqa(dev["q"], dev["r"], dev["K"], dev["V"], torch.from_numpy(sl_host).cuda())
    assert plx.get_device_status() == 0
    want = oracle.decode_gqa_ref(ref["q"], ref["r"], ref["K"], ref["V"], sl_host)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL
