"""plx_decode_noalloc, the decode entry point for callers that cannot allocate.

Some callers (a runtime that reserves all device memory up front, a
latency-critical loop that must not risk the synchronisation of cudaMalloc or
cudaFree) cannot let the library allocate its split-KV scratch.  This entry
point uses a fixed scratch array compiled into the library instead.  Its
output must match the regular entry point's (plx_decode_ex) within the bf16
parity tolerance, on two calls in a row with different shapes, and it must
not change the device's free memory after its first call.
"""
import numpy as np
import pytest
import torch

from local_linear_attention_streamed_b200 import synth
from _util import BF16_TOL, device_inputs, rel_err_rms, to_f64

pytestmark = pytest.mark.gpu


def _inputs(seed, B, H, L, d):
    t = device_inputs(seed, synth.decode_specs(B, H, L, d), synth.BF16)
    sl = torch.from_numpy(synth.seqlens(seed, B, L, ragged=True)).cuda()
    return t, sl


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
        torch.cuda.synchronize()
        free = torch.cuda.mem_get_info()[0]
        if n == 0:
            free_after_first = free
        else:
            assert free == free_after_first


def test_noalloc_scratch_holds_every_split_plan():
    """The fixed scratch (8 MiB: 128 KiB of counters, the rest partial records)
    holds the records of every split plan on this device: the split plan only
    cuts keys into chunks when the (b, h) pairs alone leave the last wave of
    CTAs underfilled, which bounds B H S.  The size check that returns
    PLX_ERR_WORKSPACE guards devices with other SM counts."""
    from local_linear_attention_streamed_b200 import plx
    cap = (8 << 20) - (128 << 10)
    for d in (64, 128):
        for L in (256, 1024, 4096, 65536):
            for bh in list(range(1, 600)) + list(range(600, 32769, 37)):
                S = plx.lib.plx_decode_num_splits(bh, 1, L, d)
                assert S >= 1
                if S > 1:
                    assert bh * S * (2 * d + 4) * 4 <= cap and bh * 4 <= (128 << 10), (d, L, bh, S)