"""Failure detection on the GPU without a fault.

Every wait in the tcgen05 prefill, backward and decode kernels is bounded in
time.  With
PLX_FAULT_INJECT=prefill_stall the TMA producer withholds the first Q/R tile,
so a barrier that nothing will complete is waited on: the kernel must give up
after its limit, report PLX_ERR_TIMEOUT through plx_get_device_status, free
its resources and leave the context usable (the next prefill is correct).
"""
import numpy as np
import pytest

import oracle
from local_linear_attention_streamed_b200 import synth
from _util import BF16_TOL, rel_err_rms, small_inputs, to_f64

pytestmark = pytest.mark.gpu


def test_prefill_timeout_is_reported_and_context_survives(monkeypatch):
    from local_linear_attention_streamed_b200 import plx
    specs = synth.prefill_specs(1, 2, 256, 128)
    dev, ref = small_inputs(31, specs, synth.BF16)
    assert plx.get_device_status() == 0
    monkeypatch.setenv("PLX_FAULT_INJECT", "prefill_stall")
    plx.prefill(dev["Q"], dev["K"], dev["V"], dev["R"], causal=True)
    assert plx.get_device_status() == -7  # PLX_ERR_TIMEOUT
    monkeypatch.delenv("PLX_FAULT_INJECT")
    out = plx.prefill(dev["Q"], dev["K"], dev["V"], dev["R"], causal=True)
    assert plx.get_device_status() == 0
    want = oracle.prefill_ref(ref["Q"], ref["K"], ref["V"], ref["R"], causal=True)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL


def test_backward_timeout_is_reported_and_context_survives(monkeypatch):
    """PLX_FAULT_INJECT=bwd_stall: one CTA of the dK/dV kernel never receives its
    K/V tiles; its bounded waits run out, the status word reports the timeout,
    and the next backward call on the same context is correct."""
    from local_linear_attention_streamed_b200 import plx
    from _util import GRAD_TOL, rel_err_fro
    B, H, N, d = 1, 2, 192, 128
    dev, ref = small_inputs(32, synth.backward_specs(B, H, N, d), synth.BF16)
    saved = plx.prefill_train(dev["Q"], dev["K"], dev["V"], dev["R"], True)
    assert plx.get_device_status() == 0
    monkeypatch.setenv("PLX_FAULT_INJECT", "bwd_stall")
    plx.prefill_backward(dev["Q"], dev["K"], dev["V"], dev["R"], *saved, dev["dO"], True)
    assert plx.get_device_status() == -7  # PLX_ERR_TIMEOUT
    monkeypatch.delenv("PLX_FAULT_INJECT")
    grads = plx.prefill_backward(dev["Q"], dev["K"], dev["V"], dev["R"], *saved, dev["dO"], True)
    assert plx.get_device_status() == 0
    want = oracle.parallax_backward_ref(ref["Q"], ref["K"], ref["V"], ref["R"], ref["dO"], True)
    for g, w in zip(grads, want):
        assert rel_err_fro(to_f64(g), w) <= GRAD_TOL


def test_decode_timeout_is_reported_and_context_survives(monkeypatch):
    """PLX_FAULT_INJECT=decode_stall: CTA 0 of the tensor-core decode never
    receives its K/V blocks; its bounded waits run out, the status word
    reports the timeout, the library clears the arrival counters that the
    unfinished (b, KV head) pairs left behind, and the next decode on the same
    context (keys split into chunks, so the counters matter) is correct."""
    import torch
    from local_linear_attention_streamed_b200 import plx
    B, Hkv, G, L, d = 1, 2, 4, 8192, 128
    H = G * Hkv
    specs = synth.decode_gqa_specs(B, H, Hkv, L, d)
    dev, ref = small_inputs(33, specs, synth.BF16)
    sl_host = np.array([L - 5], dtype=np.int32)
    sl = torch.from_numpy(sl_host).cuda()
    assert plx.get_device_status() == 0
    monkeypatch.setenv("PLX_FAULT_INJECT", "decode_stall")
    plx.decode_gqa(dev["q"], dev["r"], dev["K"], dev["V"], sl)
    assert plx.get_device_status() == -7  # PLX_ERR_TIMEOUT
    monkeypatch.delenv("PLX_FAULT_INJECT")
    want = oracle.decode_gqa_ref(ref["q"], ref["r"], ref["K"], ref["V"], sl_host)
    for _ in range(2):
        out = plx.decode_gqa(dev["q"], dev["r"], dev["K"], dev["V"], sl)
        assert plx.get_device_status() == 0
        assert rel_err_rms(to_f64(out), want) <= BF16_TOL


def test_fp8kv_decode_timeout_is_reported_and_context_survives(monkeypatch):
    """The e4m3-cache decode under PLX_FAULT_INJECT=decode_stall: CTA 0 never
    receives its code blocks, the converter and key warps' bounded waits run
    out, the timeout is reported (and the arrival counters cleared), and the
    next two decodes on the same context are correct."""
    import torch
    from local_linear_attention_streamed_b200 import plx
    B, Hkv, G, L, d = 1, 2, 4, 8192, 128
    H = G * Hkv
    specs = synth.decode_gqa_specs(B, H, Hkv, L, d)
    dev, ref = small_inputs(34, specs, synth.BF16)
    Kc, Ks = plx.kv_quantize_fp8(dev["K"])
    Vc, Vs = plx.kv_quantize_fp8(dev["V"])
    oKc, oKs = oracle.kv_quantize_fp8_ref(ref["K"])
    oVc, oVs = oracle.kv_quantize_fp8_ref(ref["V"])
    sl_host = np.array([L - 5], dtype=np.int32)
    sl = torch.from_numpy(sl_host).cuda()
    assert plx.get_device_status() == 0
    monkeypatch.setenv("PLX_FAULT_INJECT", "decode_stall")
    plx.decode_fp8kv(dev["q"], dev["r"], Kc, Ks, Vc, Vs, sl)
    assert plx.get_device_status() == -7  # PLX_ERR_TIMEOUT
    monkeypatch.delenv("PLX_FAULT_INJECT")
    want = oracle.decode_fp8kv_ref(ref["q"], ref["r"], oKc, oKs, oVc, oVs, sl_host)
    for _ in range(2):
        out = plx.decode_fp8kv(dev["q"], dev["r"], Kc, Ks, Vc, Vs, sl)
        assert plx.get_device_status() == 0
        assert rel_err_rms(to_f64(out), want) <= BF16_TOL
