"""GPU parity of the block-sparse causal prefill (plx_prefill_block_sparse)
against the float64 oracle: query i sees key j when j <= i and the (128-query
tile, 64-key block) pair is active.  Bar: bf16 max |g - o| / RMS(o_row) <= 2e-2.
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


def _mask(N, active):
    nt, nkb = (N + 127) // 128, (N + 63) // 64
    return np.array([[bool(active(t, kb)) or kb // 2 == t for kb in range(nkb)] for t in range(nt)])


def local_global(N, local_blocks=16, global_blocks=2):
    """Each tile: its diagonal blocks, the local_blocks key blocks before them and the first global_blocks."""
    return _mask(N, lambda t, kb: kb < global_blocks or 2 * t - local_blocks <= kb)


PATTERNS = {
    "all": lambda N: _mask(N, lambda t, kb: True),
    "diagonal": lambda N: _mask(N, lambda t, kb: False),
    "strided": lambda N: _mask(N, lambda t, kb: kb % 3 == 0),
    "random": lambda N: _mask(N, lambda t, kb: np.random.default_rng(t * 1000 + kb).random() < 0.4),
    "local_global": lambda N: local_global(N, 2, 1),
}


@pytest.mark.parametrize("pattern", sorted(PATTERNS))
@pytest.mark.parametrize("N,d", [(300, 128), (520, 64)])
def test_block_sparse_matches_oracle(plx, pattern, N, d):
    B, H = 1, 2
    dev, ref = small_inputs(1100 + N + len(pattern), synth.prefill_specs(B, H, N, d), synth.BF16)
    m = PATTERNS[pattern](N)
    out = plx.prefill_block_sparse(dev["Q"], dev["K"], dev["V"], dev["R"], m)
    assert plx.get_device_status() == 0
    want = oracle.prefill_block_sparse_ref(ref["Q"], ref["K"], ref["V"], ref["R"], m)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL


def _stress(d):
    B, H, N = 1, 2, 520
    dev, ref = small_inputs(13, synth.prefill_specs(B, H, N, d), synth.BF16)
    dev["K"][:, :, 200:] *= 8
    ref["K"] = dev["K"].double().cpu().numpy()
    return dev, ref, N


@pytest.mark.parametrize("d", [64, 128])
def test_block_sparse_rescale_path(plx, d):
    """Keys from position 200 on scaled by 8 (the running max jumps by far more
    than 2^8) under a local + global pattern that straddles the jump."""
    dev, ref, N = _stress(d)
    m = PATTERNS["local_global"](N)
    out = plx.prefill_block_sparse(dev["Q"], dev["K"], dev["V"], dev["R"], m)
    want = oracle.prefill_block_sparse_ref(ref["Q"], ref["K"], ref["V"], ref["R"], m)
    assert rel_err_rms(to_f64(out), want) <= BF16_TOL


def test_block_sparse_rejects_missing_diagonal(plx):
    N = 256
    x = torch.zeros((1, 1, N, 128), dtype=torch.bfloat16, device="cuda")
    m = PATTERNS["all"](N)
    m[1, 3] = False
    with pytest.raises(plx.PlxError) as e:
        plx.prefill_block_sparse(x, x, x, x, m)
    assert e.value.code == -1


def test_block_sparse_full_size_sampled(plx):
    """Local (16 blocks = 1024 keys) + global (first 2 blocks) pattern on the
    prefill workload B=8, H=16, N=4096, d=128: sampled rows."""
    B, H, N, d = 8, 16, 4096, 128
    seed = 1030
    specs = synth.prefill_specs(B, H, N, d)
    dev = device_inputs(seed, specs, synth.BF16)
    m = local_global(N)
    out = plx.prefill_block_sparse(dev["Q"], dev["K"], dev["V"], dev["R"], m)
    torch.cuda.synchronize()
    assert plx.get_device_status() == 0
    rng = np.random.default_rng(11)
    rows = [(0, 0, 0), (7, 15, N - 1), (3, 4, 1100), (5, 9, 2050)]
    rows += [(int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(N))) for _ in range(8)]
    got, want = [], []
    for (b, h, i) in rows:
        r0 = (b * H + h) * N
        keys = [j for j in range(i + 1) if m[i // 128, j // 64]]
        K = synth.host_rows_f64(seed, specs["K"], synth.BF16, r0, i + 1)[keys]
        V = synth.host_rows_f64(seed, specs["V"], synth.BF16, r0, i + 1)[keys]
        q = synth.host_rows_f64(seed, specs["Q"], synth.BF16, r0 + i, 1)[0]
        r = synth.host_rows_f64(seed, specs["R"], synth.BF16, r0 + i, 1)[0]
        want.append(oracle.parallax_row(q, r, K, V))
        got.append(to_f64(out[b, h, i]))
    assert rel_err_rms(np.stack(got), np.stack(want)) <= BF16_TOL
    assert torch.isfinite(out).all()
