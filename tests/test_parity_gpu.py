"""GPU parity: libplx.so against the float64 oracle on the same seeded inputs.

Bars: fp32 inputs
max_e |g - o| / max(|o_e|, RMS(o)) <= 1e-5; bf16 inputs max |g - o| / RMS(o)
<= 2e-2.  Small cases are compared element by element over every output;
full-size workloads on sampled outputs that the oracle recomputes from the
generator's host copy of exactly the rows it needs.
"""
import numpy as np
import pytest
import torch

import oracle
from local_linear_attention_streamed_b200 import synth
from _util import (BF16_TOL, F32_TOL, LAYER_TOL, TORCH_DT, device_inputs, rel_err_f32, rel_err_rms,
                   small_inputs, to_f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def plx():
    from local_linear_attention_streamed_b200 import plx as mod
    assert torch.cuda.is_available()
    return mod


# ---------------------------------------------------------------------------
# Generator: device fill equals the host generator bit for bit.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dist,dtype", [(synth.NORMAL, synth.BF16), (synth.NORMAL, synth.F32),
                                        (synth.RMS_ROWS, synth.BF16), (synth.RMS_ROWS, synth.F32)])
def test_device_generator_matches_host(dist, dtype):
    spec = synth.TensorSpec(synth.TID_K, (3, 5, 77, 128), dist, 0.25)
    dev = device_inputs(123, {"x": spec}, dtype)["x"].cpu()
    host = synth.host_tensor(123, spec, dtype)
    if dtype == synth.BF16:
        got = dev.view(torch.int16).numpy().view(np.uint16)
    else:
        got = dev.numpy()
    assert np.array_equal(got, host)


# ---------------------------------------------------------------------------
# Prefill.
# ---------------------------------------------------------------------------

def _prefill_case(plx, seed, B, H, N, d, dtype, causal, zero_r=False, qk_dist=synth.NORMAL):
    specs = synth.prefill_specs(B, H, N, d, qk_dist=qk_dist)
    dev, ref = small_inputs(seed, specs, dtype)
    if zero_r:
        dev["R"].zero_()
        ref["R"] = np.zeros_like(ref["R"])
    out = plx.prefill(dev["Q"], dev["K"], dev["V"], dev["R"], causal=causal)
    assert plx.get_device_status() == 0
    want = oracle.prefill_ref(ref["Q"], ref["K"], ref["V"], ref["R"], causal=causal)
    return to_f64(out), want


@pytest.mark.parametrize("zero_r", [False, True])
def test_config_tiny_fp32(plx, zero_r):
    """B=1, H=2, N=128, d=64 fp32; Q,K,V ~ N(0,1), rho ~ N(0, 0.25^2); and R = 0."""
    got, want = _prefill_case(plx, 1001, 1, 2, 128, 64, synth.F32, True, zero_r=zero_r)
    assert rel_err_f32(got, want) <= F32_TOL


def test_fp32_r_zero_is_softmax(plx):
    """With R = 0 the kernel output is softmax attention (torch SDPA in float64)."""
    specs = synth.prefill_specs(1, 2, 128, 64, qk_dist=synth.NORMAL)
    dev, ref = small_inputs(1001, specs, synth.F32)
    out = plx.prefill(dev["Q"], dev["K"], dev["V"], torch.zeros_like(dev["R"]), causal=True)
    sdpa = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(ref[n]) for n in ("Q", "K", "V")), is_causal=True).numpy()
    assert rel_err_f32(to_f64(out), sdpa) <= F32_TOL


@pytest.mark.parametrize("N,d,causal", [(1, 32, True), (77, 32, True), (200, 96, False),
                                        (129, 128, True), (257, 64, False)])
def test_fp32_shapes(plx, N, d, causal):
    got, want = _prefill_case(plx, 7, 2, 3, N, d, synth.F32, causal)
    assert rel_err_f32(got, want) <= F32_TOL


@pytest.mark.parametrize("N,d,causal", [(1, 128, True), (100, 128, True), (300, 128, True),
                                        (300, 128, False), (257, 64, True), (513, 128, True),
                                        (1, 64, True), (300, 64, False), (513, 64, True)])
def test_bf16_prefill_small(plx, N, d, causal):
    got, want = _prefill_case(plx, 11, 2, 3, N, d, synth.BF16, causal, qk_dist=synth.RMS_ROWS)
    assert rel_err_rms(got, want) <= BF16_TOL


def test_bf16_prefill_r_zero(plx):
    got, want = _prefill_case(plx, 12, 1, 2, 384, 128, synth.BF16, True, zero_r=True,
                              qk_dist=synth.RMS_ROWS)
    assert rel_err_rms(got, want) <= BF16_TOL


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
def test_bf16_prefill_rescale_path(plx, causal, d):
    """Keys from position 200 on are scaled by 8, so the running max of later
    rows jumps by far more than 2^8 after their first blocks: the kernels must
    rescale the partial O1, O2, omega and T exactly."""
    B, H, N = 1, 2, 520
    specs = synth.prefill_specs(B, H, N, d)
    dev, ref = small_inputs(13, specs, synth.BF16)
    dev["K"][:, :, 200:] *= 8
    ref["K"] = dev["K"].double().cpu().numpy()
    out = plx.prefill(dev["Q"], dev["K"], dev["V"], dev["R"], causal=causal)
    assert plx.get_device_status() == 0
    want = oracle.prefill_ref(ref["Q"], ref["K"], ref["V"], ref["R"], causal=causal)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL


def _sampled_prefill(plx, seed, B, H, N, d, rows):
    specs = synth.prefill_specs(B, H, N, d)
    dev = device_inputs(seed, specs, synth.BF16)
    out = plx.prefill(dev["Q"], dev["K"], dev["V"], dev["R"], causal=True)
    assert plx.get_device_status() == 0
    got, want = [], []
    for (b, h, i) in rows:
        r0 = (b * H + h) * N
        K = synth.host_rows_f64(seed, specs["K"], synth.BF16, r0, i + 1)
        V = synth.host_rows_f64(seed, specs["V"], synth.BF16, r0, i + 1)
        q = synth.host_rows_f64(seed, specs["Q"], synth.BF16, r0 + i, 1)[0]
        r = synth.host_rows_f64(seed, specs["R"], synth.BF16, r0 + i, 1)[0]
        want.append(oracle.parallax_row(q, r, K, V))
        got.append(out[b, h, i].double().cpu().numpy())
    return np.stack(got), np.stack(want), out


def test_prefill_compute_matched_d64_sampled(plx):
    """Head dim halved at the same width (the pages' compute-matched control):
    causal prefill B=8, H=32, N=4096, d=64 bf16, sampled rows across tiles."""
    B, H, N, d = 8, 32, 4096, 64
    rng = np.random.default_rng(4)
    rows = [(0, 0, 0), (7, 31, N - 1), (3, 17, 127), (5, 2, 128)] + \
        [(int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(N))) for _ in range(8)]
    got, want, out = _sampled_prefill(plx, 1006, B, H, N, d, rows)
    assert rel_err_rms(got, want) <= BF16_TOL
    assert torch.isfinite(out).all()


def test_config_prefill_full_size_sampled(plx):
    """Causal prefill B=8, H=16, N=4096, d=128 bf16, sampled rows across tiles."""
    B, H, N, d = 8, 16, 4096, 128
    rng = np.random.default_rng(5)
    rows = [(0, 0, 0), (0, 0, 1), (7, 15, N - 1), (3, 5, 127), (3, 5, 128), (2, 9, 2047)]
    rows += [(int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(N))) for _ in range(18)]
    got, want, out = _sampled_prefill(plx, 1004, B, H, N, d, rows)
    assert rel_err_rms(got, want) <= BF16_TOL
    assert torch.isfinite(out).all()


# ---------------------------------------------------------------------------
# Decode.
# ---------------------------------------------------------------------------

def _decode_small(plx, seed, B, H, L, d, seqlens, dtype=synth.BF16, workspace=None):
    specs = synth.decode_specs(B, H, L, d)
    dev, ref = small_inputs(seed, specs, dtype)
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    out = plx.decode(dev["q"], dev["r"], dev["K"], dev["V"], sl, workspace=workspace)
    status = plx.get_device_status()
    want = oracle.decode_ref(ref["q"], ref["r"], ref["K"], ref["V"], np.asarray(seqlens))
    return to_f64(out), want, status


@pytest.mark.parametrize("d", [64, 128])
def test_bf16_decode_ragged(plx, d):
    B, H, L = 6, 5, 1000
    seqlens = [1, 17, 256, 999, 1000, 500]
    got, want, status = _decode_small(plx, 21, B, H, L, d, seqlens)
    assert status == 0
    assert plx.lib.plx_decode_num_splits(B, H, L, d) > 1
    assert rel_err_rms(got, want) <= BF16_TOL


def test_bf16_decode_repeatable_and_user_workspace(plx):
    """Counters reset themselves: repeated calls agree; a caller workspace agrees too."""
    B, H, L, d = 4, 4, 2048, 128
    seqlens = [2048, 1500, 33, 1024]
    a, want, s1 = _decode_small(plx, 22, B, H, L, d, seqlens)
    b, _, s2 = _decode_small(plx, 22, B, H, L, d, seqlens)
    nbytes = plx.decode_workspace_bytes(B, H, L, d)
    assert nbytes > 0
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    c, _, s3 = _decode_small(plx, 22, B, H, L, d, seqlens, workspace=ws)
    assert s1 == s2 == s3 == 0
    assert np.array_equal(a, b) and np.array_equal(a, c)
    assert rel_err_rms(a, want) <= BF16_TOL


def test_bf16_decode_tensor_core_sizes_every_output(plx):
    """Sizes the tensor-core decode serves (256 (b, h) pairs, 2048 keys):
    every output, lengths at the 128-key block edges (1, 127, 128, 129, 2047,
    2048, ...) and NaN in the cache past every length, which must not leak."""
    B, H, L, d = 16, 16, 2048, 128
    specs = synth.decode_specs(B, H, L, d)
    dev, ref = small_inputs(25, specs, synth.BF16)
    seqlens = np.array([1, 2, 127, 128, 129, 255, 256, 257, 1000, 1023, 1024, 1025, 2046, 2047, 2048, 640],
                       dtype=np.int32)
    for b in range(B):
        dev["K"][b, :, seqlens[b]:] = float("nan")
        dev["V"][b, :, seqlens[b]:] = float("nan")
    out = plx.decode(dev["q"], dev["r"], dev["K"], dev["V"], torch.from_numpy(seqlens).cuda())
    assert plx.get_device_status() == 0
    assert torch.isfinite(out).all()
    want = oracle.decode_ref(ref["q"], ref["r"], ref["K"], ref["V"], seqlens)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL
    # The sliding-window form over the same cache (the last 1500 keys).
    outw = plx.decode_window(dev["q"], dev["r"], dev["K"], dev["V"], torch.from_numpy(seqlens).cuda(), 1500)
    assert plx.get_device_status() == 0
    wantw = oracle.decode_ref(ref["q"], ref["r"], ref["K"], ref["V"], seqlens, window=1500)
    assert rel_err_rms(to_f64(outw), wantw) <= BF16_TOL


@pytest.mark.parametrize("window", [None, 17000])
def test_bf16_decode_d64_head_pairs_every_output(plx, window):
    """d = 64 with H even at sizes the tensor-core decode serves (long caches,
    few heads): two heads a unit (side-by-side 64-dim halves).  Every output,
    lengths at 128-key block edges, NaN in the cache past every length."""
    B, H, L, d = 4, 8, 20480, 64
    assert plx.lib.plx_decode_uses_tc(B, H, L, d) == 1
    specs = synth.decode_specs(B, H, L, d)
    dev, ref = small_inputs(26, specs, synth.BF16)
    seqlens = np.array([1, 129, 17025, 20480], dtype=np.int32)
    for b in range(B):
        dev["K"][b, :, seqlens[b]:] = float("nan")
        dev["V"][b, :, seqlens[b]:] = float("nan")
    sl = torch.from_numpy(seqlens).cuda()
    if window is None:
        out = plx.decode(dev["q"], dev["r"], dev["K"], dev["V"], sl)
    else:
        out = plx.decode_window(dev["q"], dev["r"], dev["K"], dev["V"], sl, window)
    assert plx.get_device_status() == 0
    assert torch.isfinite(out).all()
    want = oracle.decode_ref(ref["q"], ref["r"], ref["K"], ref["V"], seqlens, window=window)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL


def test_bf16_decode_d64_head_pairs_split_keys(plx):
    """Few head pairs over long caches: chunks merged in-kernel, repeatable."""
    B, H, L, d = 1, 4, 16384, 64
    assert plx.lib.plx_decode_uses_tc(B, H, L, d) == 1 and plx.lib.plx_decode_num_splits(B, H, L, d) > 1
    got, want, status = _decode_small(plx, 27, B, H, L, d, [L - 77])
    assert status == 0
    assert rel_err_rms(got, want) <= BF16_TOL
    again, _, _ = _decode_small(plx, 27, B, H, L, d, [L - 77])
    assert np.array_equal(got, again)


def test_fp32_decode(plx):
    B, H, L, d = 3, 2, 300, 64
    got, want, status = _decode_small(plx, 23, B, H, L, d, [300, 1, 157], dtype=synth.F32)
    assert status == 0
    assert rel_err_f32(got, want) <= F32_TOL


def test_decode_bad_seqlen_reports_and_zeroes(plx):
    B, H, L, d = 4, 3, 512, 128
    specs = synth.decode_specs(B, H, L, d)
    dev, ref = small_inputs(24, specs, synth.BF16)
    sl = torch.tensor([512, 0, 513, 100], dtype=torch.int32, device="cuda")
    out = plx.decode(dev["q"], dev["r"], dev["K"], dev["V"], sl)
    assert plx.get_device_status() == -6
    assert plx.get_device_status() == 0  # the read cleared the status word
    o = to_f64(out)
    assert np.all(o[1] == 0) and np.all(o[2] == 0)
    want = oracle.decode_ref(ref["q"], ref["r"], ref["K"], ref["V"], np.array([512, 1, 1, 100]),
                             units=[(0, h) for h in range(H)] + [(3, h) for h in range(H)])
    got = np.concatenate([o[0], o[3]])
    assert rel_err_rms(got, want) <= BF16_TOL


def test_config_decode_full_size_sampled(plx):
    """Decode B=64, H=16, L=4096, d=128 bf16 (all sequences full), sampled (b, h)."""
    B, H, L, d = 64, 16, 4096, 128
    seed = 1002
    specs = synth.decode_specs(B, H, L, d)
    dev = device_inputs(seed, specs, synth.BF16)
    sl = torch.full((B,), L, dtype=torch.int32, device="cuda")
    out = plx.decode(dev["q"], dev["r"], dev["K"], dev["V"], sl)
    assert plx.get_device_status() == 0
    rng = np.random.default_rng(9)
    units = [(0, 0), (63, 15)] + [(int(rng.integers(B)), int(rng.integers(H))) for _ in range(14)]
    got, want = [], []
    for (b, h) in units:
        r0 = (b * H + h) * L
        K = synth.host_rows_f64(seed, specs["K"], synth.BF16, r0, L)
        V = synth.host_rows_f64(seed, specs["V"], synth.BF16, r0, L)
        q = synth.host_rows_f64(seed, specs["q"], synth.BF16, b * H + h, 1)[0]
        r = synth.host_rows_f64(seed, specs["r"], synth.BF16, b * H + h, 1)[0]
        want.append(oracle.parallax_row(q, r, K, V))
        got.append(out[b, h].double().cpu().numpy())
    assert rel_err_rms(np.stack(got), np.stack(want)) <= BF16_TOL
    assert torch.isfinite(out).all()


@pytest.mark.parametrize("B,L", [(1, 128), (8, 1024), (64, 4096), (256, 1024), (1, 32768),
                                 (2048, 128), (8, 16384)])
def test_config_decode_sweep_cells_sampled(plx, B, L):
    """Decode sweep cells (H=16, d=128, ragged lengths uniform on [L/2, L])."""
    H, d = 16, 128
    seed = 1003
    specs = synth.decode_specs(B, H, L, d)
    dev = device_inputs(seed, specs, synth.BF16)
    sl_host = synth.seqlens(seed, B, L, ragged=True)
    sl = torch.from_numpy(sl_host).cuda()
    out = plx.decode(dev["q"], dev["r"], dev["K"], dev["V"], sl)
    assert plx.get_device_status() == 0
    rng = np.random.default_rng(B * 7 + L)
    units = [(int(rng.integers(B)), int(rng.integers(H))) for _ in range(6)]
    got, want = [], []
    for (b, h) in units:
        n = int(sl_host[b])
        r0 = (b * H + h) * L
        K = synth.host_rows_f64(seed, specs["K"], synth.BF16, r0, n)
        V = synth.host_rows_f64(seed, specs["V"], synth.BF16, r0, n)
        q = synth.host_rows_f64(seed, specs["q"], synth.BF16, b * H + h, 1)[0]
        r = synth.host_rows_f64(seed, specs["r"], synth.BF16, b * H + h, 1)[0]
        want.append(oracle.parallax_row(q, r, K, V))
        got.append(out[b, h].double().cpu().numpy())
    assert rel_err_rms(np.stack(got), np.stack(want)) <= BF16_TOL
    del dev
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# Error paths through the ABI with real device tensors.
# ---------------------------------------------------------------------------

def test_error_codes_on_device(plx):
    x = torch.zeros(1, 2, 64, 128, dtype=torch.bfloat16, device="cuda")
    flat = torch.zeros(1 * 2 * 64 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    mis = flat[1:1 + x.numel()].view(1, 2, 64, 128)
    with pytest.raises(plx.PlxError) as e:
        plx.prefill(mis, x, x, x)
    assert e.value.code == -3
    x96 = torch.zeros(1, 2, 64, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(plx.PlxError) as e:
        plx.prefill(x96, x96, x96, x96)
    assert e.value.code == -2
    q = torch.zeros(4, 4, 128, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(4, 4, 2048, 128, dtype=torch.bfloat16, device="cuda")
    sl = torch.full((4,), 2048, dtype=torch.int32, device="cuda")
    small = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(plx.PlxError) as e:
        plx.decode(q, q, kv, kv, sl, workspace=small)
    assert e.value.code == -5
    assert plx.get_device_status() == 0


# ---------------------------------------------------------------------------
# Layer pieces and the full layer.
# ---------------------------------------------------------------------------

def test_norm_rope_matches_oracle(plx):
    B, N, H, d = 2, 300, 4, 128
    rng = np.random.default_rng(3)
    x32 = rng.standard_normal((B, N, H * d)).astype(np.float32)
    xb = torch.from_numpy(x32).to(torch.bfloat16)
    y = plx.qkr_norm_rope(xb.cuda(), H)
    xr = xb.double().numpy().reshape(B, N, H, d).transpose(0, 2, 1, 3)
    want = oracle.rope(oracle.rmsnorm(xr), np.arange(N)[None, None, :])
    assert rel_err_rms(to_f64(y), want) <= BF16_TOL


def test_config_layer_small(plx):
    """Full layer at a small width: every output row against the float64 oracle."""
    B, N, D, H = 2, 160, 256, 2
    seed = 1005
    specs = synth.layer_specs(B, N, D)
    dev, ref = small_inputs(seed, specs, synth.BF16)
    y = plx.layer_forward(dev["x"], dev["WQ"], dev["WK"], dev["WV"], dev["WR"], dev["WO"], H)
    assert plx.get_device_status() == 0
    rows = [(b, t) for b in range(B) for t in range(N)]
    want = oracle.layer_rows_ref(ref["x"], ref["WQ"], ref["WK"], ref["WV"], ref["WR"], ref["WO"], H,
                                 rows).reshape(B, N, D)
    assert rel_err_rms(to_f64(y), want) <= LAYER_TOL


def test_config_layer_full_size_sampled(plx):
    """Layer x [4, 8192, 2048], 16 heads of 128, sampled rows of two batch entries."""
    B, N, D, H = 4, 8192, 2048, 16
    seed = 1005
    specs = synth.layer_specs(B, N, D)
    dev = device_inputs(seed, specs, synth.BF16)
    y = plx.layer_forward(dev["x"], dev["WQ"], dev["WK"], dev["WV"], dev["WR"], dev["WO"], H)
    assert plx.get_device_status() == 0
    rows = [(1, 0), (1, 1), (1, 4095), (1, 8191), (3, 777), (3, 5000)]
    x = {b: synth.host_rows_f64(seed, specs["x"], synth.BF16, b * N, N) for b in (1, 3)}
    W = {n: synth.host_rows_f64(seed, specs[n], synth.BF16, 0, D) for n in ("WQ", "WK", "WV", "WR", "WO")}
    got, want = [], []
    for b in (1, 3):
        rb = [(0, t) for (bb, t) in rows if bb == b]
        want.append(oracle.layer_rows_ref(x[b][None], W["WQ"], W["WK"], W["WV"], W["WR"], W["WO"], H, rb))
        got.append(np.stack([y[b, t].double().cpu().numpy() for (_, t) in rb]))
    assert rel_err_rms(np.concatenate(got), np.concatenate(want)) <= LAYER_TOL
    assert torch.isfinite(y).all()


def test_config_layer_attention_stage_full_size(plx):
    """The attention stage of the layer workload (B=4, N=8192, 16 heads of 128)
    held to the attention bar: the bf16 q, k, v, rho the layer itself produced
    (read back from a caller workspace) go to the oracle, whose rows must match
    the layer's own attention output within BF16_TOL.  Then plx_prefill on the
    same tensors must reproduce that output bit for bit."""
    B, N, D, H = 4, 8192, 2048, 16
    d = D // H
    seed = 1005
    specs = synth.layer_specs(B, N, D)
    dev = device_inputs(seed, specs, synth.BF16)
    ws = torch.empty(plx.layer_workspace_bytes(B, N, H, d), dtype=torch.uint8, device="cuda")
    y = plx.layer_forward(dev["x"], dev["WQ"], dev["WK"], dev["WV"], dev["WR"], dev["WO"], H,
                          workspace=ws)
    assert plx.get_device_status() == 0
    assert torch.isfinite(y).all()
    v = plx.layer_workspace_views(ws, B, N, H, d)
    attn = v["attn"].clone()
    again = plx.prefill(v["q"], v["k"], v["v"], v["rho"], causal=True)
    assert plx.get_device_status() == 0
    assert torch.equal(again, attn)
    rows = [0, 1, 2, 63, 64, 127, 128, 129, 4095, 4096, 8064, 8190, 8191]
    rng = np.random.default_rng(55)
    got, want = [], []
    for (b, h) in [(0, 0), (1, 7), (3, 15)]:
        extra = [int(i) for i in rng.integers(0, N, size=6)]
        Kh, Vh = to_f64(v["k"][b, h]), to_f64(v["v"][b, h])
        qh, rh = to_f64(v["q"][b, h]), to_f64(v["rho"][b, h])
        ah = to_f64(attn[b, h])
        for i in rows + extra:
            want.append(oracle.parallax_row(qh[i], rh[i], Kh[:i + 1], Vh[:i + 1]))
            got.append(ah[i])
    assert rel_err_rms(np.stack(got), np.stack(want)) <= BF16_TOL
    del dev, ws, attn, again
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# Prefill with grouped KV heads.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("G", [2, 4, 8])
@pytest.mark.parametrize("N,d,causal", [(300, 128, True), (200, 64, True), (130, 128, False)])
def test_prefill_gqa(plx, G, N, d, causal):
    B, Hkv = 2, 2
    H = G * Hkv
    specs = synth.prefill_specs(B, H, N, d)
    specs["K"] = synth.TensorSpec(synth.TID_K, (B, Hkv, N, d), specs["K"].dist, specs["K"].sigma)
    specs["V"] = synth.TensorSpec(synth.TID_V, (B, Hkv, N, d), specs["V"].dist, specs["V"].sigma)
    dev, ref = small_inputs(1200 + G + N, specs, synth.BF16)
    out = plx.prefill_gqa(dev["Q"], dev["K"], dev["V"], dev["R"], causal=causal)
    assert plx.get_device_status() == 0
    want = oracle.prefill_gqa_ref(ref["Q"], ref["K"], ref["V"], ref["R"], causal)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL


def test_prefill_gqa_ungrouped_is_prefill(plx):
    B, H, N, d = 1, 4, 256, 128
    dev, _ = small_inputs(1210, synth.prefill_specs(B, H, N, d), synth.BF16)
    a = plx.prefill_gqa(dev["Q"], dev["K"], dev["V"], dev["R"], causal=True)
    b = plx.prefill(dev["Q"], dev["K"], dev["V"], dev["R"], causal=True)
    assert torch.equal(a, b)
