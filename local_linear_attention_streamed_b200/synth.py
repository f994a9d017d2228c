"""Seeded synthetic inputs for Parallax attention, identical on host and device.

This module holds no Parallax arithmetic.  It defines one counter-based
generator and draws every tensor of the workloads from it, so that the float64
CPU oracle (which regenerates any slice it needs on the host with numpy) and
the CUDA path (which fills multi-GB caches on the device with the
``plx_synth_*`` kernels of ``libplx_synth.so``) see bit-identical values.

Generator (the same definition is written out in ``csrc/synth.cu``):

* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014; finaliser constants as published by Vigna):
  ``mix(z) = z ^ z>>30; *0xBF58476D1CE4E5B9; ^ >>27; *0x94D049BB133111EB; ^ >>31``.
  The stream of a tensor is keyed by ``key = mix(seed*256 + tensor_id)`` and
  element ``c`` (flat row-major index) draws ``h = mix(key + (c+1)*0x9E3779B97F4A7C15)``
  (the c-th output of a SplitMix64 generator seeded with ``key``).
* Approximately normal deviate from the Irwin-Hall sum of the four 16-bit
  lanes of ``h``: ``n = sum(lanes) - 2*65535`` (an integer, |n| <= 131070,
  mean 0, standard deviation 65536/sqrt(3)).  ``NORMAL`` stores
  ``float64(n) * scale`` with ``scale = sigma*sqrt(3)/65536``; ``RMS_ROWS``
  stores ``float64(n) / sqrt(sum_row(n^2) / d)`` (each length-d row has unit
  RMS before rounding), where the row sum of squares is an exact int64.
* Rounding: float64 -> float32 (round to nearest even), then, for bf16
  tensors, float32 -> bf16 by round-to-nearest-even on the bit pattern.
  Every step is a single IEEE operation or integer arithmetic, so numpy and
  CUDA agree bit for bit.

The deviates have the mean, variance and symmetry of N(0, sigma^2) but a
bounded support of +-3.46 sigma; the pages specify only "N(0,1)" and
"RMS-normalised rows", which this matches to the precision that matters for
the kernels' numerics and performance.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
M1 = np.uint64(0xBF58476D1CE4E5B9)
M2 = np.uint64(0x94D049BB133111EB)
MASK16 = np.uint64(0xFFFF)

# Distribution codes shared with csrc/synth.cu.
NORMAL = 0
RMS_ROWS = 1

# dtype codes shared with the C ABI (PLX_F32 / PLX_BF16).
F32 = 0
BF16 = 1

# Tensor ids: one independent stream per tensor of a workload.
TID_Q, TID_K, TID_V, TID_R, TID_SEQLENS = 1, 2, 3, 4, 5
TID_DO = 6
TID_X, TID_WQ, TID_WK, TID_WV, TID_WR, TID_WO = 11, 12, 13, 14, 15, 16


def _mix(z):
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * M1
        z = (z ^ (z >> np.uint64(27))) * M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tensor_id: int) -> int:
    """64-bit key of the stream that tensor ``tensor_id`` of ``seed`` draws from."""
    z = np.uint64((int(seed) * 256 + int(tensor_id)) & 0xFFFFFFFFFFFFFFFF)
    return int(_mix(z))


def raw_hash(key: int, idx: np.ndarray) -> np.ndarray:
    """SplitMix64 output number ``idx`` (uint64 array) of the stream seeded by ``key``."""
    idx = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + (idx + np.uint64(1)) * GAMMA
    return _mix(z)


def irwin_hall(key: int, idx: np.ndarray) -> np.ndarray:
    """Integer deviate n = sum of the four 16-bit lanes of the hash - 2*65535 (int64)."""
    h = raw_hash(key, idx)
    s = (h & MASK16) + ((h >> np.uint64(16)) & MASK16) + ((h >> np.uint64(32)) & MASK16) + (h >> np.uint64(48))
    return s.astype(np.int64) - 2 * 65535


def normal_scale(sigma: float) -> float:
    """Multiplier that maps the Irwin-Hall integer to a deviate of std ``sigma``."""
    return float(sigma) * math.sqrt(3.0) / 65536.0


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern (uint16), round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return (u >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact upcast of bf16 bit patterns to float64."""
    u = np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def draw_f64(seed: int, tensor_id: int, start: int, count: int, dist: int,
             sigma: float = 1.0, row: int = 0) -> np.ndarray:
    """Unrounded float64 deviates for flat elements [start, start+count).

    For RMS_ROWS, ``row`` is the row length and ``start``/``count`` must be
    multiples of it.
    """
    key = stream_key(seed, tensor_id)
    idx = np.arange(start, start + count, dtype=np.uint64)
    n = irwin_hall(key, idx)
    if dist == NORMAL:
        return n.astype(np.float64) * normal_scale(sigma)
    if dist == RMS_ROWS:
        if row <= 0 or start % row or count % row:
            raise ValueError("RMS_ROWS needs whole rows")
        nr = n.reshape(-1, row)
        ss = (nr * nr).sum(axis=1)  # exact: |n| < 2^18, row <= 2^12
        den = np.sqrt(ss.astype(np.float64) / float(row))
        return (nr.astype(np.float64) / den[:, None]).reshape(-1)
    raise ValueError(f"unknown distribution {dist}")


def draw(seed: int, tensor_id: int, start: int, count: int, dist: int, dtype: int,
         sigma: float = 1.0, row: int = 0) -> np.ndarray:
    """Stored values: float32 array for F32, uint16 bf16 bit patterns for BF16."""
    x32 = draw_f64(seed, tensor_id, start, count, dist, sigma, row).astype(np.float32)
    if dtype == F32:
        return x32
    if dtype == BF16:
        return f32_to_bf16_bits(x32)
    raise ValueError(f"unknown dtype {dtype}")


def stored_to_f64(arr: np.ndarray, dtype: int) -> np.ndarray:
    """Exact float64 value of stored elements (what the oracle consumes)."""
    if dtype == F32:
        return np.asarray(arr, dtype=np.float32).astype(np.float64)
    return bf16_bits_to_f64(arr)


def seqlens(seed: int, B: int, L: int, ragged: bool) -> np.ndarray:
    """Per-sequence KV lengths: all L, or uniform on {ceil(L/2), ..., L}."""
    if not ragged:
        return np.full(B, L, dtype=np.int32)
    lo = (L + 1) // 2
    span = L - lo + 1
    h = raw_hash(stream_key(seed, TID_SEQLENS), np.arange(B, dtype=np.uint64))
    return (lo + (h % np.uint64(span)).astype(np.int64)).astype(np.int32)


# ---------------------------------------------------------------------------
# Workload recipes (shapes and distributions of the pages' workloads).
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class TensorSpec:
    tensor_id: int
    shape: tuple
    dist: int
    sigma: float = 1.0

    @property
    def numel(self) -> int:
        n = 1
        for s in self.shape:
            n *= s
        return n

    @property
    def row(self) -> int:
        return self.shape[-1]


def prefill_specs(B, H, N, d, qk_dist=RMS_ROWS, rho_sigma=0.25):
    """Q, K, V, R for a prefill: q, k RMS rows (or N(0,1)), v ~ N(0,1), rho ~ N(0, rho_sigma^2)."""
    shp = (B, H, N, d)
    return {
        "Q": TensorSpec(TID_Q, shp, qk_dist),
        "K": TensorSpec(TID_K, shp, qk_dist),
        "V": TensorSpec(TID_V, shp, NORMAL, 1.0),
        "R": TensorSpec(TID_R, shp, NORMAL, rho_sigma),
    }


def decode_specs(B, H, L, d, rho_sigma=0.25):
    """q, r [B,H,d]; Kcache, Vcache [B,H,L,d]."""
    return {
        "q": TensorSpec(TID_Q, (B, H, d), RMS_ROWS),
        "K": TensorSpec(TID_K, (B, H, L, d), RMS_ROWS),
        "V": TensorSpec(TID_V, (B, H, L, d), NORMAL, 1.0),
        "r": TensorSpec(TID_R, (B, H, d), NORMAL, rho_sigma),
    }


def backward_specs(B, H, N, d, qk_dist=RMS_ROWS, rho_sigma=0.25):
    """prefill_specs plus the output gradient dO ~ N(0, 1), all [B, H, N, d]."""
    specs = prefill_specs(B, H, N, d, qk_dist=qk_dist, rho_sigma=rho_sigma)
    specs["dO"] = TensorSpec(TID_DO, (B, H, N, d), NORMAL, 1.0)
    return specs


def decode_gqa_specs(B, H, Hkv, L, d, rho_sigma=0.25):
    """Grouped KV heads: q, r [B,H,d]; Kcache, Vcache [B,Hkv,L,d] (same distributions as decode)."""
    return {
        "q": TensorSpec(TID_Q, (B, H, d), RMS_ROWS),
        "K": TensorSpec(TID_K, (B, Hkv, L, d), RMS_ROWS),
        "V": TensorSpec(TID_V, (B, Hkv, L, d), NORMAL, 1.0),
        "r": TensorSpec(TID_R, (B, H, d), NORMAL, rho_sigma),
    }


def layer_specs(B, N, D):
    """x ~ N(0,1) [B,N,D]; W_Q, W_K, W_V, W_R, W_O ~ N(0, 1/D) stored [in, out]."""
    ws = 1.0 / math.sqrt(D)
    return {
        "x": TensorSpec(TID_X, (B, N, D), NORMAL, 1.0),
        "WQ": TensorSpec(TID_WQ, (D, D), NORMAL, ws),
        "WK": TensorSpec(TID_WK, (D, D), NORMAL, ws),
        "WV": TensorSpec(TID_WV, (D, D), NORMAL, ws),
        "WR": TensorSpec(TID_WR, (D, D), NORMAL, ws),
        "WO": TensorSpec(TID_WO, (D, D), NORMAL, ws),
    }


def host_tensor(seed: int, spec: TensorSpec, dtype: int) -> np.ndarray:
    """Whole tensor on the host (stored representation), shaped like ``spec``."""
    return draw(seed, spec.tensor_id, 0, spec.numel, spec.dist, dtype, spec.sigma,
                spec.row).reshape(spec.shape)


def host_rows_f64(seed: int, spec: TensorSpec, dtype: int, row_start: int, nrows: int) -> np.ndarray:
    """Exact float64 of rows [row_start, row_start+nrows) of the flattened [-1, d] tensor."""
    d = spec.row
    st = draw(seed, spec.tensor_id, row_start * d, nrows * d, spec.dist, dtype, spec.sigma, d)
    return stored_to_f64(st, dtype).reshape(nrows, d)


# ---------------------------------------------------------------------------
# Device fill through libplx_synth.so (plain C ABI, see include/plx_synth.h).
# ---------------------------------------------------------------------------

_synth_lib = None


def _lib():
    global _synth_lib
    if _synth_lib is None:
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libplx_synth.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run __graft_entry__.build() first")
        lib = ctypes.CDLL(path)
        lib.plx_synth_fill.restype = ctypes.c_int
        lib.plx_synth_fill.argtypes = [
            ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64, ctypes.c_uint64,
            ctypes.c_int, ctypes.c_double, ctypes.c_int64, ctypes.c_void_p]
        _synth_lib = lib
    return _synth_lib


def device_fill(ptr: int, dtype: int, seed: int, spec: TensorSpec, stream: int = 0) -> None:
    """Fill ``spec.numel`` elements at device pointer ``ptr`` with the stream of ``spec``."""
    scale = normal_scale(spec.sigma) if spec.dist == NORMAL else 0.0
    rc = _lib().plx_synth_fill(ctypes.c_void_p(ptr), dtype,
                               ctypes.c_uint64(stream_key(seed, spec.tensor_id)),
                               ctypes.c_uint64(spec.numel), spec.dist, scale,
                               ctypes.c_int64(spec.row), ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"plx_synth_fill failed with code {rc}")
