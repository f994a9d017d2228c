"""GPU parity of the training forward (saved statistics) and of the backward
pass, through the C ABI, against the float64 oracle on the same seeded inputs.

Bars.  The training forward's out is the inference kernel's out bit for bit;
vbar (fp32, from the bf16 weights of the value MMAs) is held to the forward's
bf16 bar (max |g - o| / RMS of the row <= 2e-2); lse and tbar are fp32 results
of fp32 sums over bf16 inputs (bar 1e-4 of max(1, |lse|) and 1e-3 of
max(1, RMS(t))).  Each whole gradient tensor is held to a relative Frobenius
error <= GRAD_TOL and a largest elementwise error
max_e |g - o| / max(|o_e|, RMS(o)) <= GRAD_MAX_TOL (derived in tests/_util.py
and checked attainable in tests/test_backward_bound.py).  The backward kernels
are checked twice: given the oracle's saved tensors (their own error alone),
and after the training forward (the composition a user runs).
"""
import numpy as np
import pytest
import torch

import oracle
from local_linear_attention_streamed_b200 import synth
from _util import (BF16_TOL, GRAD_MAX_TOL, GRAD_TOL, device_inputs, rel_err_elem, rel_err_fro, rel_err_rms,
                   small_inputs, to_f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def plx():
    from local_linear_attention_streamed_b200 import plx as mod
    assert torch.cuda.is_available()
    return mod


def _check_grads(grads, want, where=""):
    for name, g, w in zip(("dQ", "dK", "dV", "dR"), grads, want):
        assert torch.isfinite(g).all(), (name, where)
        gf = to_f64(g).reshape(w.shape)
        if not np.any(w):
            # A single visible key: out = v_0 whatever q, k and rho are, so
            # dQ, dK and dR are exactly zero; the kernels leave the fp32
            # rounding residue of dA - F (inputs are O(1)).
            assert np.max(np.abs(gf)) <= 1e-3, (name, where)
            continue
        fro, emax = rel_err_fro(gf, w), rel_err_elem(gf, w)
        assert fro <= GRAD_TOL and emax <= GRAD_MAX_TOL, (name, where, fro, emax)


def _case(plx, seed, B, H, N, d, causal):
    specs = synth.backward_specs(B, H, N, d)
    dev, ref = small_inputs(seed, specs, synth.BF16)
    out, vbar, lse, tbar = plx.prefill_train(dev["Q"], dev["K"], dev["V"], dev["R"], causal)
    grads = plx.prefill_backward(dev["Q"], dev["K"], dev["V"], dev["R"], out, vbar, lse, tbar, dev["dO"], causal)
    torch.cuda.synchronize()
    assert plx.get_device_status() == 0
    return dev, ref, (out, vbar, lse, tbar), grads


@pytest.mark.parametrize("N,d,causal", [(320, 128, True), (200, 64, False), (1, 128, True)])
def test_train_forward_saved_statistics(plx, N, d, causal):
    B, H = 2, 3
    dev, ref, (out, vbar, lse, tbar), _ = _case(plx, 300 + N, B, H, N, d, causal)
    plain = plx.prefill(dev["Q"], dev["K"], dev["V"], dev["R"], causal=causal)
    assert torch.equal(out, plain)
    w_vbar, w_lse, w_tbar = oracle.prefill_stats_ref(ref["Q"], ref["K"], ref["V"], ref["R"], causal)
    assert rel_err_rms(to_f64(vbar), w_vbar) <= BF16_TOL
    assert np.max(np.abs(to_f64(lse) - w_lse) / np.maximum(1.0, np.abs(w_lse))) <= 1e-4
    t_rms = np.sqrt(np.mean((ref["R"] * ref["K"]).sum(-1) ** 2)) * np.sqrt(N)
    assert np.max(np.abs(to_f64(tbar) - w_tbar)) <= 1e-3 * max(1.0, t_rms)


CASES = [(64, 128, True), (200, 128, True), (320, 128, False), (384, 128, True),
         (256, 64, True), (200, 64, False), (130, 64, True), (1, 128, True), (1, 64, False)]


@pytest.mark.parametrize("N,d,causal", CASES)
def test_backward_kernels_match_oracle(plx, N, d, causal):
    """The backward kernels alone, fed the oracle's saved tensors (out rounded
    to bf16 as the forward stores it): every element of dQ, dK, dV, dR over
    several 64/128-row tiles, ragged tails (N not a multiple of 64 or 128), a
    single key, causal and full."""
    B, H = 1, 2
    specs = synth.backward_specs(B, H, N, d)
    dev, ref = small_inputs(500 + N + d, specs, synth.BF16)
    vbar, lse, tbar = oracle.prefill_stats_ref(ref["Q"], ref["K"], ref["V"], ref["R"], causal)
    out = oracle.prefill_ref(ref["Q"], ref["K"], ref["V"], ref["R"], causal=causal)
    cuda = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()
    grads = plx.prefill_backward(dev["Q"], dev["K"], dev["V"], dev["R"], cuda(out, torch.bfloat16),
                                 cuda(vbar, torch.float32), cuda(lse, torch.float32), cuda(tbar, torch.float32),
                                 dev["dO"], causal)
    torch.cuda.synchronize()
    assert plx.get_device_status() == 0
    want = oracle.parallax_backward_ref(ref["Q"], ref["K"], ref["V"], ref["R"], ref["dO"], causal)
    _check_grads(grads, want)


@pytest.mark.parametrize("N,d,causal", CASES)
def test_train_forward_then_backward_matches_oracle(plx, N, d, causal):
    """The composition a user runs: training forward, then the backward pass."""
    B, H = 1, 2
    _, ref, _, grads = _case(plx, 500 + N + d, B, H, N, d, causal)
    want = oracle.parallax_backward_ref(ref["Q"], ref["K"], ref["V"], ref["R"], ref["dO"], causal)
    _check_grads(grads, want)


def test_backward_caller_workspace_and_autograd(plx):
    B, H, N, d = 1, 2, 192, 128
    specs = synth.backward_specs(B, H, N, d)
    dev, ref = small_inputs(77, specs, synth.BF16)
    ws = torch.empty(plx.prefill_bwd_workspace_bytes(B, H, N, d) // 4, dtype=torch.float32, device="cuda")
    out, vbar, lse, tbar = plx.prefill_train(dev["Q"], dev["K"], dev["V"], dev["R"], True)
    g1 = plx.prefill_backward(dev["Q"], dev["K"], dev["V"], dev["R"], out, vbar, lse, tbar, dev["dO"], True,
                              workspace=ws)
    leaves = [dev[n].clone().requires_grad_(True) for n in "QKVR"]
    o2 = plx.parallax_attention(*leaves, causal=True)
    o2.backward(dev["dO"])
    assert torch.equal(o2.detach(), out)
    for a, leaf in zip(g1, leaves):
        assert torch.equal(a, leaf.grad)


def test_backward_rejects_bad_arguments(plx):
    B, H, N, d = 1, 1, 64, 96
    x = torch.zeros((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    vb = torch.zeros((B, H, N, d), dtype=torch.float32, device="cuda")
    s = torch.zeros((B, H, N), dtype=torch.float32, device="cuda")
    with pytest.raises(plx.PlxError) as e:
        plx.prefill_backward(x, x, x, x, x, vb, s, s, x, True)
    assert e.value.code == -2
    d = 128
    x = torch.zeros((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    vb = torch.zeros((B, H, N, d), dtype=torch.float32, device="cuda")
    ws = torch.empty(16, dtype=torch.float32, device="cuda")
    with pytest.raises(plx.PlxError) as e:
        plx.prefill_backward(x, x, x, x, x, vb, s, s, x, True, workspace=ws)
    assert e.value.code == -5


def test_backward_full_size_heads(plx):
    """Causal B=8, H=16, N=4096, d=128 (the prefill workload), in the launch
    configuration the benchmark times; two whole heads (heads are independent)
    compared element by element with the oracle run on those heads alone."""
    B, H, N, d = 8, 16, 4096, 128
    seed = 1010
    specs = synth.backward_specs(B, H, N, d)
    dev = device_inputs(seed, specs, synth.BF16)
    out, vbar, lse, tbar = plx.prefill_train(dev["Q"], dev["K"], dev["V"], dev["R"], True)
    grads = plx.prefill_backward(dev["Q"], dev["K"], dev["V"], dev["R"], out, vbar, lse, tbar, dev["dO"], True)
    torch.cuda.synchronize()
    assert plx.get_device_status() == 0
    for g in grads:
        assert torch.isfinite(g).all()
    for (b, h) in [(0, 0), (7, 13)]:
        row0 = (b * H + h) * N
        head = {n: synth.host_rows_f64(seed, specs[n], synth.BF16, row0, N).reshape(1, 1, N, d)
                for n in ("Q", "K", "V", "R", "dO")}
        want = oracle.parallax_backward_ref(head["Q"], head["K"], head["V"], head["R"], head["dO"], True)
        _check_grads([g[b, h] for g in grads], [w[0, 0] for w in want], where=(b, h))


def test_calls_from_a_fresh_thread(plx):
    """The library binds the device's context in every call, so a thread that
    has made no CUDA call of its own (an autograd worker, a data loader) can
    call it after another thread did (the tensor maps need a current context)."""
    import threading
    B, H, N, d = 1, 2, 128, 128
    dev, _ = small_inputs(88, synth.backward_specs(B, H, N, d), synth.BF16)
    saved = plx.prefill_train(dev["Q"], dev["K"], dev["V"], dev["R"], True)
    first = plx.prefill_backward(dev["Q"], dev["K"], dev["V"], dev["R"], *saved, dev["dO"], True)
    res = {}

    def work():
        try:
            res["g"] = plx.prefill_backward(dev["Q"], dev["K"], dev["V"], dev["R"], *saved, dev["dO"], True)
            res["o"] = plx.prefill(dev["Q"], dev["K"], dev["V"], dev["R"], causal=True)
            torch.cuda.synchronize()
        except Exception as e:  # reported below
            res["e"] = e

    t = threading.Thread(target=work)
    t.start()
    t.join()
    assert "e" not in res, res.get("e")
    for a, b in zip(first, res["g"]):
        assert torch.equal(a, b)
    assert torch.equal(res["o"], saved[0])


@pytest.mark.parametrize("N,d,W", [(300, 128, 37), (300, 128, 100), (320, 128, 200), (260, 64, 64),
                                   (200, 64, 150), (130, 128, 1)])
def test_window_backward_matches_oracle(plx, N, d, W):
    """Sliding-window training forward then backward: every gradient element,
    windows shorter and longer than the 64/128-row blocks, ragged N."""
    B, H = 1, 2
    dev, ref = small_inputs(600 + N + W, synth.backward_specs(B, H, N, d), synth.BF16)
    saved = plx.prefill_train(dev["Q"], dev["K"], dev["V"], dev["R"], True, window=W)
    grads = plx.prefill_backward(dev["Q"], dev["K"], dev["V"], dev["R"], *saved, dev["dO"], True, window=W)
    torch.cuda.synchronize()
    assert plx.get_device_status() == 0
    out_w = plx.prefill_window(dev["Q"], dev["K"], dev["V"], dev["R"], W)
    assert torch.equal(saved[0], out_w)
    want = oracle.parallax_backward_ref(ref["Q"], ref["K"], ref["V"], ref["R"], ref["dO"], True, window=W)
    _check_grads(grads, want, where=W)


def _gqa_specs(B, H, Hkv, N, d):
    specs = synth.backward_specs(B, H, N, d)
    for n, tid in (("K", synth.TID_K), ("V", synth.TID_V)):
        specs[n] = synth.TensorSpec(tid, (B, Hkv, N, d), specs[n].dist, specs[n].sigma)
    return specs


@pytest.mark.parametrize("G,N,d,causal", [(2, 200, 128, True), (4, 320, 128, True), (8, 130, 128, False),
                                          (4, 256, 64, True), (2, 200, 64, False), (8, 1, 128, True)])
def test_gqa_train_then_backward_matches_oracle(plx, G, N, d, causal):
    """Grouped KV heads (query head h reads KV head h / G): the training
    forward's out equals the grouped inference prefill bit for bit, and every
    element of dQ, dR (per query head) and of dK, dV (per KV head, summed over
    the group's query heads) meets the gradient bars; ragged N, causal and full."""
    B, Hkv = 2, 2
    H = G * Hkv
    dev, ref = small_inputs(1400 + 10 * G + N + d, _gqa_specs(B, H, Hkv, N, d), synth.BF16)
    saved = plx.prefill_train(dev["Q"], dev["K"], dev["V"], dev["R"], causal)
    grads = plx.prefill_backward(dev["Q"], dev["K"], dev["V"], dev["R"], *saved, dev["dO"], causal)
    torch.cuda.synchronize()
    assert plx.get_device_status() == 0
    assert torch.equal(saved[0], plx.prefill_gqa(dev["Q"], dev["K"], dev["V"], dev["R"], causal=causal))
    assert grads[1].shape == dev["K"].shape and grads[2].shape == dev["V"].shape
    want = oracle.parallax_backward_ref(ref["Q"], ref["K"], ref["V"], ref["R"], ref["dO"], causal)
    _check_grads(grads, want, where=G)


def test_gqa_autograd_matches_direct_calls(plx):
    B, H, Hkv, N, d = 1, 8, 2, 192, 128
    dev, _ = small_inputs(1450, _gqa_specs(B, H, Hkv, N, d), synth.BF16)
    saved = plx.prefill_train(dev["Q"], dev["K"], dev["V"], dev["R"], True)
    g1 = plx.prefill_backward(dev["Q"], dev["K"], dev["V"], dev["R"], *saved, dev["dO"], True)
    leaves = [dev[n].clone().requires_grad_(True) for n in "QKVR"]
    o2 = plx.parallax_attention(*leaves, causal=True)
    o2.backward(dev["dO"])
    assert torch.equal(o2.detach(), saved[0])
    for a, leaf in zip(g1, leaves):
        assert torch.equal(a, leaf.grad)


def test_gqa_backward_rejects_bad_groups(plx):
    B, N, d = 1, 64, 128
    q = torch.zeros((B, 6, N, d), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((B, 4, N, d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        plx.prefill_train(q, kv, kv, q, True)
    with pytest.raises(ValueError):  # K and V of different head counts
        plx.prefill_train(q, kv, kv[:, :2].contiguous(), q, True)


def test_gqa_backward_full_size_group(plx):
    """B=2, H=32, Hkv=8, N=4096, d=128 causal: the whole group of KV head
    (1, 5) (its four query heads' dQ, dR and the head's dK, dV) compared element
    by element with the oracle run on that group alone."""
    B, H, Hkv, N, d = 2, 32, 8, 4096, 128
    G = H // Hkv
    seed = 1460
    specs = _gqa_specs(B, H, Hkv, N, d)
    dev = device_inputs(seed, specs, synth.BF16)
    saved = plx.prefill_train(dev["Q"], dev["K"], dev["V"], dev["R"], True)
    grads = plx.prefill_backward(dev["Q"], dev["K"], dev["V"], dev["R"], *saved, dev["dO"], True)
    torch.cuda.synchronize()
    assert plx.get_device_status() == 0
    for g in grads:
        assert torch.isfinite(g).all()
    b, hk = 1, 5
    qrows = lambda n: synth.host_rows_f64(seed, specs[n], synth.BF16, (b * H + hk * G) * N, G * N).reshape(1, G, N, d)
    krows = lambda n: synth.host_rows_f64(seed, specs[n], synth.BF16, (b * Hkv + hk) * N, N).reshape(1, 1, N, d)
    head = {n: qrows(n) for n in ("Q", "R", "dO")}
    head.update({n: krows(n) for n in ("K", "V")})
    want = oracle.parallax_backward_ref(head["Q"], head["K"], head["V"], head["R"], head["dO"], True)
    got = [grads[0][b, hk * G:(hk + 1) * G], grads[1][b, hk:hk + 1], grads[2][b, hk:hk + 1],
           grads[3][b, hk * G:(hk + 1) * G]]
    _check_grads(got, [w[0] for w in want], where=(b, hk))


@pytest.mark.parametrize("G,N,d,W", [(2, 300, 128, 37), (4, 320, 128, 128), (4, 260, 64, 64), (8, 200, 128, 150)])
def test_gqa_window_prefill_and_backward(plx, G, N, d, W):
    """Grouped KV heads with a sliding window: the inference prefill against
    the oracle on the KV heads repeated over each group, the training forward
    equal to it bit for bit, and every gradient element (dK, dV per KV head,
    summed over the group) against the oracle's."""
    B, Hkv = 1, 2
    H = G * Hkv
    dev, ref = small_inputs(1500 + 10 * G + W, _gqa_specs(B, H, Hkv, N, d), synth.BF16)
    out = plx.prefill_gqa(dev["Q"], dev["K"], dev["V"], dev["R"], window=W)
    assert plx.get_device_status() == 0
    Kr, Vr = (np.repeat(ref[n], G, axis=1) for n in ("K", "V"))
    want = oracle.prefill_ref(ref["Q"], Kr, Vr, ref["R"], window=W)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL
    saved = plx.prefill_train(dev["Q"], dev["K"], dev["V"], dev["R"], True, window=W)
    assert torch.equal(saved[0], out)
    grads = plx.prefill_backward(dev["Q"], dev["K"], dev["V"], dev["R"], *saved, dev["dO"], True, window=W)
    torch.cuda.synchronize()
    assert plx.get_device_status() == 0
    assert grads[1].shape == dev["K"].shape
    wgrads = oracle.parallax_backward_ref(ref["Q"], ref["K"], ref["V"], ref["R"], ref["dO"], True, window=W)
    _check_grads(grads, wgrads, where=(G, W))
