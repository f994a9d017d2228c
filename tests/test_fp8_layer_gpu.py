"""GPU parity of the layer with dynamic fp8 linears (plx_layer_forward_fp8)
against the float64 oracle with the same per-tensor e4m3 quantisation.

Bars, element by element over every output (derived in tests/_util.py;
tests/test_fp8_layer_bound.py shows both are attainable and that unquantised
linears, one wrong attention tile and one wrong head fail them): per element
max_e |g - o| / RMS(o_row) <= FP8_LAYER_ELEM_TOL, per output row
RMS(g - o) / RMS(o) <= FP8_LAYER_ROW_TOL.
"""
import pytest
import torch

import oracle
from local_linear_attention_streamed_b200 import synth
from _util import FP8_LAYER_ELEM_TOL, FP8_LAYER_ROW_TOL, rel_err_row, rel_err_rms, small_inputs, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def plx():
    from local_linear_attention_streamed_b200 import plx as mod
    assert torch.cuda.is_available()
    return mod


@pytest.mark.parametrize("B,N,D,H", [(2, 160, 256, 2), (2, 160, 256, 4), (1, 320, 512, 4)])
def test_fp8_layer_matches_oracle(plx, B, N, D, H):
    dev, ref = small_inputs(40 + D + H, synth.layer_specs(B, N, D), synth.BF16)
    y = plx.layer_forward_fp8(dev["x"], dev["WQ"], dev["WK"], dev["WV"], dev["WR"], dev["WO"], H)
    assert plx.get_device_status() == 0
    want = oracle.layer_fp8_ref(*[ref[n] for n in ("x", "WQ", "WK", "WV", "WR", "WO")], H)
    assert torch.isfinite(y).all()
    got = to_f64(y)
    assert rel_err_rms(got, want) <= FP8_LAYER_ELEM_TOL
    assert rel_err_row(got, want) <= FP8_LAYER_ROW_TOL


def test_fp8_layer_caller_workspace_and_bad_sizes(plx):
    B, N, D, H = 1, 64, 256, 2
    dev, _ = small_inputs(5, synth.layer_specs(B, N, D), synth.BF16)
    ws = torch.empty(int(plx.lib.plx_layer_fp8_workspace_bytes(B, N, H, D // H)), dtype=torch.uint8, device="cuda")
    a = plx.layer_forward_fp8(dev["x"], dev["WQ"], dev["WK"], dev["WV"], dev["WR"], dev["WO"], H, workspace=ws)
    b = plx.layer_forward_fp8(dev["x"], dev["WQ"], dev["WK"], dev["WV"], dev["WR"], dev["WO"], H)
    assert torch.equal(a, b)
    x = dev["x"][:, :63].contiguous()
    with pytest.raises(plx.PlxError) as e:
        plx.layer_forward_fp8(x, dev["WQ"], dev["WK"], dev["WV"], dev["WR"], dev["WO"], H)
    assert e.value.code == -2


def test_fp8_layer_full_config(plx):
    """The layer workload x[4, 8192, 2048], 16 heads of 128: finite, and within a
    few percent (relative Frobenius) of the bf16 layer, as fp8 linears predict
    (the oracle cannot run the whole layer at this size)."""
    B, N, D, H = 4, 8192, 2048, 16
    specs = synth.layer_specs(B, N, D)
    from _util import device_inputs
    t = device_inputs(31, specs, synth.BF16)
    y8 = plx.layer_forward_fp8(t["x"], t["WQ"], t["WK"], t["WV"], t["WR"], t["WO"], H)
    y16 = plx.layer_forward(t["x"], t["WQ"], t["WK"], t["WV"], t["WR"], t["WO"], H)
    assert plx.get_device_status() == 0
    assert torch.isfinite(y8).all()
    rel = float((y8.float() - y16.float()).norm() / y16.float().norm())
    assert 1e-3 < rel < 0.2, rel
