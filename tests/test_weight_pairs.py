"""The decodes carry each weight w and w t as a bf16 hi + lo pair (hi =
bf16(x), lo = bf16(x - hi), both round to nearest even) as columns of the
value product.  Checked on the CPU: the pair holds x to within 2^-16 of x over
the whole fp32 range the weights take (w in (0, 2^8] under the lazy running
max, times any t), and a single bf16 operand does not (2^-9)."""
import numpy as np
import torch


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def test_hi_lo_pairs_hold_sixteen_bits():
    rng = np.random.default_rng(11)
    w = 2.0 ** rng.uniform(-40, 8, 200000)                       # lazy max: w <= 2^8
    t = rng.standard_normal(200000) * 20.0
    for x in (w, w * t):
        x = x.astype(np.float32)
        hi = _bf16(x)
        lo = _bf16(x.astype(np.float64) - hi)
        rel2 = np.abs((hi.astype(np.float64) + lo) - x) / np.abs(x)
        rel1 = np.abs(hi.astype(np.float64) - x) / np.abs(x)
        assert rel2.max() <= 2.0 ** -16
        assert rel1.max() > 2.0 ** -10
