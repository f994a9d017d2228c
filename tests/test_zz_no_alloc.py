"""plx_decode_noalloc, the decode entry point for callers that cannot allocate.

Some callers (a runtime that reserves all device memory up front, a
latency-critical loop that must not risk the synchronisation of cudaMalloc or
cudaFree) cannot let the library allocate its split-KV scratch.  This entry
point uses a fixed scratch array compiled into the library instead.  Its
output must match the float64 oracle and the regular entry point's
(plx_decode_ex) within the bf16 parity tolerance, on two calls in a row with
different shapes, and it must not change the device's free memory after its
first call.
"""
import numpy as np
import pytest
import torch

import oracle
from local_linear_attention_streamed_b200 import synth
from _util import BF16_TOL, device_inputs, rel_err_rms, to_f64

pytestmark = pytest.mark.gpu


def _inputs(seed, B, H, L, d):
    t = device_inputs(seed, synth.decode_specs(B, H, L, d), synth.BF16)
    sl = torch.from_numpy(synth.seqlens(seed, B, L, ragged=True)).cuda()
    return t, sl


def _oracle_units(seed, B, H, L, d, units):
    """Oracle outputs of (b, h) units, from the generator's host copy of exactly their rows."""
    specs = synth.decode_specs(B, H, L, d)
    sl = synth.seqlens(seed, B, L, ragged=True)
    want = []
    for (b, h) in units:
        n = int(sl[b])
        r0 = (b * H + h) * L
        K = synth.host_rows_f64(seed, specs["K"], synth.BF16, r0, n)
        V = synth.host_rows_f64(seed, specs["V"], synth.BF16, r0, n)
        q = synth.host_rows_f64(seed, specs["q"], synth.BF16, b * H + h, 1)[0]
        r = synth.host_rows_f64(seed, specs["r"], synth.BF16, b * H + h, 1)[0]
        want.append(oracle.parallax_row(q, r, K, V))
    return np.stack(want)


def test_noalloc_matches_regular_decode_on_two_calls():
    from local_linear_attention_streamed_b200 import plx
    cases = [(41, 16, 16, 4096, 128), (42, 4, 8, 2048, 64)]
    prepared = []
    for (seed, B, H, L, d) in cases:
        assert plx.lib.plx_decode_num_splits(B, H, L, d) > 1  # the scratch is really used
        t, sl = _inputs(seed, B, H, L, d)
        ref = plx.decode(t["q"], t["r"], t["K"], t["V"], sl)
        assert plx.get_device_status() == 0
        prepared.append((t, sl, to_f64(ref)))
    torch.cuda.synchronize()
    free_after_first = None
    for n, (t, sl, ref) in enumerate(prepared):
        out = torch.empty_like(t["q"])
        plx.decode_noalloc(t["q"], t["r"], t["K"], t["V"], sl, out=out)
        assert plx.get_device_status() == 0
        got = to_f64(out)
        assert np.isfinite(got).all()
        assert rel_err_rms(got, ref) <= BF16_TOL
        seed, B, H, L, d = cases[n]
        rng = np.random.default_rng(seed)
        units = [(0, 0), (B - 1, H - 1)] + [(int(rng.integers(B)), int(rng.integers(H))) for _ in range(10)]
        want = _oracle_units(seed, B, H, L, d, units)
        assert rel_err_rms(np.stack([got[b, h] for (b, h) in units]), want) <= BF16_TOL
        torch.cuda.synchronize()
        free = torch.cuda.mem_get_info()[0]
        if n == 0:
            free_after_first = free
        else:
            assert free == free_after_first


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from local_linear_attention_streamed_b200 import plx
    B, H, L, d = 250, 16, 1024, 128  # 4000 (b, h) x 3 splits of fp32 records > 8 MiB
    S = plx.lib.plx_decode_num_splits(B, H, L, d)
    assert S > 1 and B * H * S * (2 * d + 4) * 4 > (8 << 20) - (128 << 10)
    small = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    sl = torch.ones(B, dtype=torch.int32, device="cuda")
    rc = plx.lib.plx_decode_noalloc(small.data_ptr(), small.data_ptr(), small.data_ptr(),
                                    small.data_ptr(), sl.data_ptr(), small.data_ptr(), B, H, L, d,
                                    None)
    assert rc == -5
    assert plx.get_device_status() == 0
