"""Thin ctypes binding over libplx.so (include/plx.h).

Argument marshalling only: torch tensors are passed as raw device pointers and
the current torch stream; every step of the computation runs in the library's
CUDA kernels.  Loading fails loudly when the library is missing; there is no
fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

PLX_F32 = 0
PLX_BF16 = 1
PLX_ERR_CUDA = -4

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libplx.so")

# Exported symbols and their C signatures (mirrors include/plx.h).
_vp, _i, _sz, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
SIGNATURES = {
    "plx_prefill": (_i, [_vp] * 5 + [_i] * 5),
    "plx_prefill_ex": (_i, [_vp] * 5 + [_i] * 6 + [_vp]),
    "plx_decode": (_i, [_vp] * 6 + [_i] * 4),
    "plx_decode_ex": (_i, [_vp] * 6 + [_i] * 5 + [_vp, _sz, _vp]),
    "plx_decode_workspace_bytes": (_sz, [_i] * 4),
    "plx_decode_num_splits": (_i, [_i] * 4),
    "plx_decode_uses_tc": (_i, [_i] * 4),
    "plx_decode_noalloc": (_i, [_vp] * 6 + [_i] * 4 + [_vp]),
    "plx_decode_gqa": (_i, [_vp] * 6 + [_i] * 5 + [_vp, _sz, _vp]),
    "plx_decode_gqa_workspace_bytes": (_sz, [_i] * 5),
    "plx_qkr_norm_rope": (_i, [_vp, _vp] + [_i] * 4 + [_f, _f, _vp]),
    "plx_layer_workspace_bytes": (_sz, [_i] * 4),
    "plx_layer_forward": (_i, [_vp] * 7 + [_i] * 4 + [_vp, _sz, _vp]),
    "plx_layer_fp8_workspace_bytes": (_sz, [_i] * 4),
    "plx_layer_forward_fp8": (_i, [_vp] * 7 + [_i] * 4 + [_vp, _sz, _vp]),
    "plx_prefill_window": (_i, [_vp] * 5 + [_i] * 6 + [_vp]),
    "plx_prefill_block_sparse": (_i, [_vp] * 5 + [_i] * 4 + [_vp, _vp]),
    "plx_prefill_gqa": (_i, [_vp] * 5 + [_i] * 6 + [_vp]),
    "plx_decode_window": (_i, [_vp] * 6 + [_i] * 7 + [_vp, _sz, _vp]),
    "plx_decode_window_workspace_bytes": (_sz, [_i] * 6),
    "plx_prefill_train": (_i, [_vp] * 8 + [_i] * 5 + [_vp]),
    "plx_prefill_bwd_workspace_bytes": (_sz, [_i] * 4),
    "plx_prefill_bwd": (_i, [_vp] * 13 + [_i] * 5 + [_vp, _sz, _vp]),
    "plx_prefill_train_window": (_i, [_vp] * 8 + [_i] * 5 + [_vp]),
    "plx_prefill_bwd_window": (_i, [_vp] * 13 + [_i] * 5 + [_vp, _sz, _vp]),
    "plx_prefill_train_gqa": (_i, [_vp] * 8 + [_i] * 6 + [_vp]),
    "plx_prefill_train_ex": (_i, [_vp] * 8 + [_i] * 7 + [_vp]),
    "plx_prefill_bwd_ex": (_i, [_vp] * 13 + [_i] * 7 + [_vp, _sz, _vp]),
    "plx_prefill_gqa_window": (_i, [_vp] * 5 + [_i] * 6 + [_vp]),
    "plx_prefill_bwd_gqa": (_i, [_vp] * 13 + [_i] * 6 + [_vp, _sz, _vp]),
    "plx_prefill_dilated": (_i, [_vp] * 5 + [_i] * 7 + [_vp]),
    "plx_kv_quantize_fp8": (_i, [_vp, _vp, _vp, ctypes.c_longlong, _i, _vp]),
    "plx_decode_fp8kv_workspace_bytes": (_sz, [_i] * 5),
    "plx_decode_fp8kv": (_i, [_vp] * 8 + [_i] * 5 + [_vp, _sz, _vp]),
    "plx_get_device_status": (_i, [_vp]),
    "plx_status_string": (ctypes.c_char_p, [_i]),
    "plx_last_cuda_error": (ctypes.c_char_p, []),
    "plx_abi_version": (_i, []),
}


class PlxError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = f"{where}: {status_string(code)} (code {code})"
        if code == PLX_ERR_CUDA:
            msg += f": {lib.plx_last_cuda_error().decode()}"
        super().__init__(msg)
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with __graft_entry__.build() "
                           "(python -m local_linear_attention_streamed_b200._build)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def status_string(code: int) -> str:
    return lib.plx_status_string(int(code)).decode()


def _check(rc: int, where: str) -> None:
    if rc != 0:
        raise PlxError(rc, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return PLX_BF16
    if t.dtype == torch.float32:
        return PLX_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _dev(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def prefill(Q, K, V, R, causal: bool = True, out=None, stream=None):
    """Parallax prefill over [B, H, N, d] tensors (bf16 or fp32); returns out."""
    B, H, N, d = Q.shape
    for n, t in (("K", K), ("V", V), ("R", R)):
        if t.shape != Q.shape or t.dtype != Q.dtype:
            raise ValueError(f"{n} must match Q in shape and dtype")
    if out is None:
        out = torch.empty_like(Q)
    rc = lib.plx_prefill_ex(_dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(R, "R"), _dev(out, "out"),
                            B, H, N, d, int(bool(causal)), _dtype_code(Q), _stream_ptr(stream))
    _check(rc, "plx_prefill_ex")
    return out


def prefill_window(Q, K, V, R, window: int, out=None, stream=None):
    """Sliding-window causal prefill (query i sees its last `window` keys); returns out."""
    B, H, N, d = Q.shape
    for n, t in (("K", K), ("V", V), ("R", R)):
        if t.shape != Q.shape or t.dtype != Q.dtype:
            raise ValueError(f"{n} must match Q in shape and dtype")
    if out is None:
        out = torch.empty_like(Q)
    rc = lib.plx_prefill_window(_dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(R, "R"), _dev(out, "out"),
                                B, H, N, d, int(window), _dtype_code(Q), _stream_ptr(stream))
    _check(rc, "plx_prefill_window")
    return out


def prefill_gqa(Q, K, V, R, causal: bool = True, out=None, stream=None, window=None):
    """bf16 prefill with grouped KV heads: Q, R [B, H, N, d]; K, V [B, Hkv, N, d]
    (``window``: the last W keys of each query, as prefill_window)."""
    B, H, N, d = Q.shape
    Hkv = K.shape[1]
    if K.shape != (B, Hkv, N, d) or V.shape != K.shape or R.shape != Q.shape:
        raise ValueError("K, V must be [B, Hkv, N, d] and R like Q")
    if out is None:
        out = torch.empty_like(Q)
    if window is None:
        rc = lib.plx_prefill_gqa(_dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(R, "R"), _dev(out, "out"),
                                 B, H, Hkv, N, d, int(bool(causal)), _stream_ptr(stream))
        _check(rc, "plx_prefill_gqa")
    else:
        rc = lib.plx_prefill_gqa_window(_dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(R, "R"), _dev(out, "out"),
                                        B, H, Hkv, N, d, int(window), _stream_ptr(stream))
        _check(rc, "plx_prefill_gqa_window")
    return out


def prefill_block_sparse(Q, K, V, R, block_mask, out=None, stream=None):
    """Block-sparse causal prefill: ``block_mask`` is a host array [ceil(N/128), ceil(N/64)]
    (truthy = the 64-key block is visible to the 128-query tile); returns out."""
    import numpy as np
    B, H, N, d = Q.shape
    for n, t in (("K", K), ("V", V), ("R", R)):
        if t.shape != Q.shape or t.dtype != Q.dtype:
            raise ValueError(f"{n} must match Q in shape and dtype")
    m = np.ascontiguousarray(np.asarray(block_mask).astype(np.uint8))
    if m.shape != ((N + 127) // 128, (N + 63) // 64):
        raise ValueError("block_mask must be [ceil(N/128), ceil(N/64)]")
    if out is None:
        out = torch.empty_like(Q)
    rc = lib.plx_prefill_block_sparse(_dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(R, "R"), _dev(out, "out"),
                                      B, H, N, d, m.ctypes.data, _stream_ptr(stream))
    _check(rc, "plx_prefill_block_sparse")
    return out


def decode_window(q, r, Kcache, Vcache, seqlens, window: int, out=None, workspace=None, stream=None):
    """Sliding-window decode step: each query sees the last `window` keys of its sequence.

    Kcache/Vcache are [B, Hkv, L, d] with H a multiple of Hkv (Hkv == H: one KV head per head).
    """
    B, H, d = q.shape
    Hkv, L = Kcache.shape[1], Kcache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    ws, wsb = (0, 0) if workspace is None else (_dev(workspace, "workspace"),
                                                workspace.numel() * workspace.element_size())
    rc = lib.plx_decode_window(_dev(q, "q"), _dev(r, "r"), _dev(Kcache, "Kcache"), _dev(Vcache, "Vcache"),
                               _dev(seqlens, "seqlens"), _dev(out, "out"), B, H, Hkv, L, d, int(window),
                               _dtype_code(q), ws, wsb, _stream_ptr(stream))
    _check(rc, "plx_decode_window")
    return out


def _kv_heads(Q, K, V):
    """KV heads of K and V ([B, Hkv, N, d], H a multiple of Hkv)."""
    B, H, N, d = Q.shape
    Hkv = K.shape[1]
    if K.shape != (B, Hkv, N, d) or V.shape != K.shape or Hkv < 1 or H % Hkv:
        raise ValueError("K, V must be [B, Hkv, N, d] with H a multiple of Hkv")
    return Hkv


def prefill_train(Q, K, V, R, causal: bool = True, stream=None, window=None):
    """bf16 prefill that also saves the backward pass's inputs (``window``:
    the sliding-window prefill of prefill_window).  K and V may have fewer
    heads than Q (grouped KV heads, as prefill_gqa).

    Returns (out, vbar, lse, tbar): out bf16 [B, H, N, d], vbar fp32
    [B, H, N, d], lse and tbar fp32 [B, H, N] (see plx_prefill_train in
    include/plx.h).
    """
    B, H, N, d = Q.shape
    Hkv = _kv_heads(Q, K, V)
    for n, t in (("K", K), ("V", V), ("R", R)):
        if t.dtype != Q.dtype:
            raise ValueError(f"{n} must match Q's dtype")
    if R.shape != Q.shape:
        raise ValueError("R must match Q's shape")
    if Q.dtype != torch.bfloat16:
        raise TypeError("prefill_train takes bf16 tensors")
    out = torch.empty_like(Q)
    vbar = torch.empty(Q.shape, dtype=torch.float32, device=Q.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=Q.device)
    tbar = torch.empty((B, H, N), dtype=torch.float32, device=Q.device)
    if Hkv != H:
        rc = lib.plx_prefill_train_ex(_dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(R, "R"), _dev(out, "out"),
                                      _dev(vbar, "vbar"), _dev(lse, "lse"), _dev(tbar, "tbar"), B, H, Hkv, N, d,
                                      int(bool(causal)), 0 if window is None else int(window), _stream_ptr(stream))
        _check(rc, "plx_prefill_train_ex")
    elif window is None:
        rc = lib.plx_prefill_train(_dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(R, "R"), _dev(out, "out"),
                                   _dev(vbar, "vbar"), _dev(lse, "lse"), _dev(tbar, "tbar"), B, H, N, d,
                                   int(bool(causal)), _stream_ptr(stream))
        _check(rc, "plx_prefill_train")
    else:
        rc = lib.plx_prefill_train_window(_dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(R, "R"),
                                          _dev(out, "out"), _dev(vbar, "vbar"), _dev(lse, "lse"),
                                          _dev(tbar, "tbar"), B, H, N, d, int(window), _stream_ptr(stream))
        _check(rc, "plx_prefill_train_window")
    return out, vbar, lse, tbar


def prefill_bwd_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(lib.plx_prefill_bwd_workspace_bytes(B, H, N, d))


def prefill_backward(Q, K, V, R, out, vbar, lse, tbar, dO, causal: bool = True, grads=None,
                     workspace=None, stream=None, window=None):
    """Gradients (dQ, dK, dV, dR) of sum(out * dO) for one bf16 prefill.

    ``out, vbar, lse, tbar`` are what prefill_train returned for the same
    inputs; ``grads`` optionally gives the four output tensors.  With grouped
    KV heads (K, V [B, Hkv, N, d]) dK and dV have K's shape: each sums over
    its group's query heads.
    """
    B, H, N, d = Q.shape
    Hkv = _kv_heads(Q, K, V)
    for n, t in (("K", K), ("V", V)):
        if t.dtype != torch.bfloat16:
            raise ValueError(f"{n} must be bf16")
    for n, t in (("R", R), ("out", out), ("dO", dO)):
        if t.shape != Q.shape or t.dtype != torch.bfloat16:
            raise ValueError(f"{n} must be bf16 of Q's shape")
    if vbar.shape != Q.shape or vbar.dtype != torch.float32:
        raise ValueError("vbar must be fp32 of Q's shape")
    for n, t in (("lse", lse), ("tbar", tbar)):
        if t.shape != (B, H, N) or t.dtype != torch.float32:
            raise ValueError(f"{n} must be fp32 [B, H, N]")
    if grads is None:
        grads = (torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V), torch.empty_like(Q))
    dQ, dK, dV, dR = grads
    ws, wsb = (0, 0) if workspace is None else (_dev(workspace, "workspace"),
                                                workspace.numel() * workspace.element_size())
    args = (_dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(R, "R"), _dev(out, "out"), _dev(vbar, "vbar"),
            _dev(lse, "lse"), _dev(tbar, "tbar"), _dev(dO, "dO"), _dev(dQ, "dQ"), _dev(dK, "dK"),
            _dev(dV, "dV"), _dev(dR, "dR"), B, H, N, d)
    if Hkv != H:
        rc = lib.plx_prefill_bwd_ex(*args[:14], H, Hkv, N, d, int(bool(causal)), 0 if window is None else int(window),
                                    ws, wsb, _stream_ptr(stream))
        _check(rc, "plx_prefill_bwd_ex")
    elif window is None:
        rc = lib.plx_prefill_bwd(*args, int(bool(causal)), ws, wsb, _stream_ptr(stream))
        _check(rc, "plx_prefill_bwd")
    else:
        rc = lib.plx_prefill_bwd_window(*args, int(window), ws, wsb, _stream_ptr(stream))
        _check(rc, "plx_prefill_bwd_window")
    return dQ, dK, dV, dR


class ParallaxAttention(torch.autograd.Function):
    """Autograd wrapper: forward = prefill_train, backward = prefill_backward (bf16)."""

    @staticmethod
    def forward(ctx, Q, K, V, R, causal=True, window=None):
        Q, K, V, R = (t.contiguous() for t in (Q, K, V, R))
        out, vbar, lse, tbar = prefill_train(Q, K, V, R, causal, window=window)
        ctx.save_for_backward(Q, K, V, R, out, vbar, lse, tbar)
        ctx.causal = causal
        ctx.window = window
        return out

    @staticmethod
    def backward(ctx, dO):
        Q, K, V, R, out, vbar, lse, tbar = ctx.saved_tensors
        dQ, dK, dV, dR = prefill_backward(Q, K, V, R, out, vbar, lse, tbar,
                                          dO.contiguous().to(torch.bfloat16), ctx.causal, window=ctx.window)
        return dQ, dK, dV, dR, None, None


def parallax_attention(Q, K, V, R, causal: bool = True, window=None):
    """Differentiable bf16 Parallax attention over [B, H, N, d] (d in {64, 128});
    ``window`` (None or W >= 1) makes it the sliding-window prefill; K and V
    may have fewer heads (grouped KV heads, with or without a window)."""
    return ParallaxAttention.apply(Q, K, V, R, causal, window)


def decode_workspace_bytes(B: int, H: int, L: int, d: int) -> int:
    return int(lib.plx_decode_workspace_bytes(B, H, L, d))


def decode(q, r, Kcache, Vcache, seqlens, out=None, workspace=None, stream=None):
    """One decode step: q, r [B, H, d]; caches [B, H, L, d]; seqlens int32 [B]."""
    B, H, L, d = Kcache.shape
    if q.shape != (B, H, d) or r.shape != (B, H, d) or Vcache.shape != Kcache.shape:
        raise ValueError("shape mismatch")
    if seqlens.dtype != torch.int32 or seqlens.shape != (B,):
        raise ValueError("seqlens must be int32 [B]")
    if out is None:
        out = torch.empty_like(q)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    rc = lib.plx_decode_ex(_dev(q, "q"), _dev(r, "r"), _dev(Kcache, "Kcache"), _dev(Vcache, "Vcache"),
                           _dev(seqlens, "seqlens"), _dev(out, "out"), B, H, L, d, _dtype_code(q),
                           ws_ptr, ws_bytes, _stream_ptr(stream))
    _check(rc, "plx_decode_ex")
    return out


def decode_noalloc(q, r, Kcache, Vcache, seqlens, out=None, stream=None):
    """As decode() for bf16, through plx_decode_noalloc: no device memory is allocated
    (the library's fixed scratch array is used)."""
    B, H, L, d = Kcache.shape
    if q.shape != (B, H, d) or r.shape != (B, H, d) or Vcache.shape != Kcache.shape:
        raise ValueError("shape mismatch")
    if seqlens.dtype != torch.int32 or seqlens.shape != (B,):
        raise ValueError("seqlens must be int32 [B]")
    if out is None:
        out = torch.empty_like(q)
    rc = lib.plx_decode_noalloc(_dev(q, "q"), _dev(r, "r"), _dev(Kcache, "Kcache"),
                                _dev(Vcache, "Vcache"), _dev(seqlens, "seqlens"), _dev(out, "out"),
                                B, H, L, d, _stream_ptr(stream))
    _check(rc, "plx_decode_noalloc")
    return out


def decode_gqa(q, r, Kcache, Vcache, seqlens, out=None, workspace=None, stream=None):
    """One bf16 decode step with grouped KV heads: q, r [B, H, d]; caches [B, Hkv, L, d]
    (query head h reads KV head h // (H // Hkv)); seqlens int32 [B]."""
    B, Hkv, L, d = Kcache.shape
    H = q.shape[1]
    if q.shape != (B, H, d) or r.shape != (B, H, d) or Vcache.shape != Kcache.shape:
        raise ValueError("shape mismatch")
    if seqlens.dtype != torch.int32 or seqlens.shape != (B,):
        raise ValueError("seqlens must be int32 [B]")
    if out is None:
        out = torch.empty_like(q)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    rc = lib.plx_decode_gqa(_dev(q, "q"), _dev(r, "r"), _dev(Kcache, "Kcache"), _dev(Vcache, "Vcache"),
                            _dev(seqlens, "seqlens"), _dev(out, "out"), B, H, Hkv, L, d,
                            ws_ptr, ws_bytes, _stream_ptr(stream))
    _check(rc, "plx_decode_gqa")
    return out


def prefill_dilated(Q, K, V, R, dilation: int, window: int = 0, out=None, stream=None):
    """Dilated causal prefill: query i sees keys i, i - r, i - 2r, ... (the last
    ``window`` of them; all when 0).  Q, R [B, H, N, d]; K, V [B, Hkv, N, d]."""
    B, H, N, d = Q.shape
    Hkv = K.shape[1]
    if out is None:
        out = torch.empty_like(Q)
    rc = lib.plx_prefill_dilated(_dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(R, "R"), _dev(out, "out"),
                                 B, H, Hkv, N, d, dilation, window, _stream_ptr(stream))
    _check(rc, "plx_prefill_dilated")
    return out


def kv_quantize_fp8(X, codes=None, scales=None, stream=None):
    """Per-row dynamic e4m3 quantisation of bf16 cache rows X[..., d]:
    returns (codes uint8 [..., d], scales float32 [...])."""
    d = X.shape[-1]
    rows = X.numel() // d
    if codes is None:
        codes = torch.empty(X.shape, dtype=torch.uint8, device=X.device)
    if scales is None:
        scales = torch.empty(X.shape[:-1], dtype=torch.float32, device=X.device)
    rc = lib.plx_kv_quantize_fp8(_dev(X, "X"), _dev(codes, "codes"), _dev(scales, "scales"), rows, d,
                                 _stream_ptr(stream))
    _check(rc, "plx_kv_quantize_fp8")
    return codes, scales


def decode_fp8kv_workspace_bytes(B: int, H: int, Hkv: int, L: int, d: int) -> int:
    return int(lib.plx_decode_fp8kv_workspace_bytes(B, H, Hkv, L, d))


def decode_fp8kv(q, r, Kcodes, Kscales, Vcodes, Vscales, seqlens, out=None, workspace=None, stream=None):
    """Decode over an e4m3 cache: q, r bf16 [B, H, d]; codes uint8 [B, Hkv, L, d];
    scales float32 [B, Hkv, L]; seqlens int32 [B]."""
    B, H, d = q.shape
    Hkv, L = Kcodes.shape[1], Kcodes.shape[2]
    if out is None:
        out = torch.empty_like(q)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    rc = lib.plx_decode_fp8kv(_dev(q, "q"), _dev(r, "r"), _dev(Kcodes, "Kcodes"), _dev(Kscales, "Kscales"),
                              _dev(Vcodes, "Vcodes"), _dev(Vscales, "Vscales"), _dev(seqlens, "seqlens"),
                              _dev(out, "out"), B, H, Hkv, L, d, ws_ptr, ws_bytes, _stream_ptr(stream))
    _check(rc, "plx_decode_fp8kv")
    return out


def qkr_norm_rope(x, H: int, eps: float = 1e-6, base: float = 10000.0, out=None, stream=None):
    """x bf16 [B, N, H*d] -> RoPE(RMSNorm(.)) per head as [B, H, N, d]."""
    B, N, D = x.shape
    d = D // H
    if out is None:
        out = torch.empty((B, H, N, d), dtype=x.dtype, device=x.device)
    rc = lib.plx_qkr_norm_rope(_dev(x, "x"), _dev(out, "out"), B, N, H, d, eps, base,
                               _stream_ptr(stream))
    _check(rc, "plx_qkr_norm_rope")
    return out


def layer_forward(x, WQ, WK, WV, WR, WO, H: int, out=None, workspace=None, stream=None):
    """Full Parallax attention layer: x bf16 [B, N, H*d], W* bf16 [H*d, H*d] stored [in, out]."""
    B, N, D = x.shape
    d = D // H
    if out is None:
        out = torch.empty_like(x)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    rc = lib.plx_layer_forward(_dev(x, "x"), _dev(WQ, "WQ"), _dev(WK, "WK"), _dev(WV, "WV"),
                               _dev(WR, "WR"), _dev(WO, "WO"), _dev(out, "out"), B, N, H, d,
                               ws_ptr, ws_bytes, _stream_ptr(stream))
    _check(rc, "plx_layer_forward")
    return out


def layer_workspace_bytes(B: int, N: int, H: int, d: int) -> int:
    return int(lib.plx_layer_workspace_bytes(B, N, H, d))


def layer_workspace_views(workspace, B: int, N: int, H: int, d: int) -> dict:
    """Views of a caller workspace after plx_layer_forward returned: the layer's
    own bf16 attention inputs q, k, v, rho and its attention output, each
    [B, H, N, d] (the slots the header lists)."""
    slot = -(-(B * N * H * d * 2) // 256) * 256
    assert workspace.dtype == torch.uint8 and workspace.numel() >= 9 * slot
    def view(i):
        return workspace[i * slot:i * slot + B * N * H * d * 2].view(torch.bfloat16).view(B, H, N, d)
    return {"q": view(4), "k": view(5), "v": view(6), "rho": view(7), "attn": view(8)}


def layer_forward_fp8(x, WQ, WK, WV, WR, WO, H: int, out=None, workspace=None, stream=None):
    """The layer of layer_forward with its five linears in dynamic per-tensor fp8 (e4m3)."""
    B, N, D = x.shape
    d = D // H
    if out is None:
        out = torch.empty_like(x)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    rc = lib.plx_layer_forward_fp8(_dev(x, "x"), _dev(WQ, "WQ"), _dev(WK, "WK"), _dev(WV, "WV"),
                                   _dev(WR, "WR"), _dev(WO, "WO"), _dev(out, "out"), B, N, H, d,
                                   ws_ptr, ws_bytes, _stream_ptr(stream))
    _check(rc, "plx_layer_forward_fp8")
    return out


def get_device_status(stream=None) -> int:
    """Synchronises the stream, returns and clears the device status code."""
    return int(lib.plx_get_device_status(_stream_ptr(stream)))
