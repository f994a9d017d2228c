"""C ABI of libplx.so on the CPU: it loads, exports what include/*.h declares,
and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "local_linear_attention_streamed_b200")


def _declared(header):
    text = open(os.path.join(ROOT, "include", header)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(plx_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from local_linear_attention_streamed_b200 import plx
    return plx.lib


@pytest.mark.parametrize("header,so", [("plx.h", "libplx.so"), ("plx_synth.h", "libplx_synth.so")])
def test_exports_every_declared_symbol(header, so):
    names = _declared(header)
    assert names, header
    dll = ctypes.CDLL(os.path.join(PKG, so))
    missing = [n for n in names if not hasattr(dll, n)]
    assert not missing, f"{so} lacks {missing}"


def test_binding_covers_header(lib):
    from local_linear_attention_streamed_b200 import plx
    assert set(_declared("plx.h")) == set(plx.SIGNATURES)


def test_version_and_status_strings(lib):
    assert lib.plx_abi_version() == 1
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        s = lib.plx_status_string(code).decode()
        assert s and s != "unknown status code"
    assert lib.plx_status_string(-99).decode() == "unknown status code"


A = 0x10000  # aligned fake device addresses: validation fails before they are used


def test_prefill_rejects_bad_arguments(lib):
    ok = [A, A, A, A, A]
    assert lib.plx_prefill_ex(None, A, A, A, A, 1, 1, 8, 64, 1, 1, None) == -1
    assert lib.plx_prefill_ex(*ok, 0, 1, 8, 64, 1, 1, None) == -1
    assert lib.plx_prefill_ex(*ok, 1, 1, 0, 64, 1, 1, None) == -1
    assert lib.plx_prefill_ex(*ok, 1, 1, 8, 64, 1, 7, None) == -1
    assert lib.plx_prefill_ex(*ok, 1, 1, 8, 96, 1, 1, None) == -2   # bf16 needs d in {64, 128}
    assert lib.plx_prefill_ex(*ok, 1, 1, 8, 160, 1, 0, None) == -2  # f32 needs d <= 128
    assert lib.plx_prefill_ex(*ok, 1, 1, 8, 48, 1, 0, None) == -2   # f32 needs d % 32 == 0
    assert lib.plx_prefill_ex(A, A + 2, A, A, A, 1, 1, 8, 64, 1, 1, None) == -3


def test_decode_rejects_bad_arguments(lib):
    ok = [A] * 6
    assert lib.plx_decode_ex(A, A, A, A, None, A, 1, 1, 8, 128, 1, None, 0, None) == -1
    assert lib.plx_decode_ex(*ok, 1, 0, 8, 128, 1, None, 0, None) == -1
    assert lib.plx_decode_ex(*ok, 1, 1, 8, 32, 1, None, 0, None) == -2
    assert lib.plx_decode_ex(A, A, A, A + 8, A, A, 1, 1, 8, 128, 1, None, 0, None) == -3
    assert lib.plx_decode_ex(A, A, A, A, A + 2, A, 1, 1, 8, 128, 1, None, 0, None) == -3


def test_decode_size_bounds_are_shared(lib):
    """Every decode entry point rejects the same oversized problems on the host:
    more than 2^24 query (b, h) pairs, or cache rows (B * KV heads * L) that
    reach 2^31 once a 128-key block is added."""
    ok = [A] * 6
    big_bh = (1 << 24) // 16 + 1
    assert lib.plx_decode_ex(*ok, big_bh, 16, 8, 128, 1, None, 0, None) == -2
    assert lib.plx_decode_noalloc(*ok, big_bh, 16, 8, 128, None) == -2
    rows_L = ((1 << 31) - 128) // 64       # B * Hkv = 64: B*Hkv*L + 128 just reaches 2^31
    assert lib.plx_decode_ex(*ok, 4, 16, rows_L, 128, 1, None, 0, None) == -2
    assert lib.plx_decode_noalloc(*ok, 4, 16, rows_L, 128, None) == -2
    assert lib.plx_decode_gqa(*ok, 4, 64, 16, rows_L, 128, None, 0, None) == -2
    assert lib.plx_decode_window(*ok, 4, 64, 16, rows_L, 128, 1024, 1, None, 0, None) == -2


def test_decode_gqa_rejects_bad_arguments(lib):
    ok = [A] * 6
    assert lib.plx_decode_gqa(A, A, A, A, None, A, 1, 8, 2, 64, 128, None, 0, None) == -1
    assert lib.plx_decode_gqa(*ok, 1, 8, 3, 64, 128, None, 0, None) == -1   # H not a multiple of Hkv
    assert lib.plx_decode_gqa(*ok, 1, 6, 2, 64, 128, None, 0, None) == -2   # group of 3
    assert lib.plx_decode_gqa(*ok, 1, 32, 2, 64, 128, None, 0, None) == -2  # group of 16
    assert lib.plx_decode_gqa(*ok, 1, 8, 2, 64, 96, None, 0, None) == -2
    assert lib.plx_decode_gqa(A, A, A, A + 8, A, A, 1, 8, 2, 64, 128, None, 0, None) == -3
    assert lib.plx_decode_gqa_workspace_bytes(1, 8, 3, 64, 128) == 0
    # Two (b, KV head) pairs over 8192 keys: the split plan takes the most
    # chunks it allows (L / 256) for one or two CTAs per SM alike, so the
    # ungrouped plan of the same pairs gives the grouped decode's count.
    S = lib.plx_decode_num_splits(1, 2, 8192, 128)
    assert S > 1
    assert lib.plx_decode_gqa_workspace_bytes(1, 8, 2, 8192, 128) == 8 * S * (2 * 128 + 4) * 4
    assert lib.plx_decode_gqa_workspace_bytes(1, 16, 2, 8192, 128) > 0


def test_decode_kernel_choice(lib):
    """The ungrouped bf16 decode's size rule, as plx_decode_uses_tc reports it
    (1 = tensor-core kernel, 0 = warp-MMA kernel): at d = 128 long caches,
    or enough (b, h) with medium ones; at d = 64 head pairs for long caches
    over few heads only."""
    cells = {(64, 16, 4096, 128): 1, (1, 16, 32768, 128): 1, (8, 16, 4096, 128): 0,
             (64, 16, 1024, 128): 1, (256, 16, 16384, 128): 1, (2048, 16, 128, 128): 0,
             (16, 16, 2048, 128): 1, (8, 16, 2048, 128): 0, (256, 16, 1024, 128): 0,
             (1, 32, 32768, 64): 1, (64, 32, 4096, 64): 0, (1, 31, 32768, 64): 0, (4, 32, 16384, 64): 0}
    for (B, H, L, d), want in cells.items():
        assert lib.plx_decode_uses_tc(B, H, L, d) == want, (B, H, L, d)
    assert lib.plx_decode_uses_tc(1, 16, 4096, 96) == -1


def test_fp8_cache_calls_reject_bad_arguments(lib):
    # plx_kv_quantize_fp8(X, codes, scales, rows, d, stream)
    assert lib.plx_kv_quantize_fp8(None, A, A, 4, 128, None) == -1
    assert lib.plx_kv_quantize_fp8(A, A, A, 0, 128, None) == -1
    assert lib.plx_kv_quantize_fp8(A, A, A, 4, 96, None) == -2
    assert lib.plx_kv_quantize_fp8(A + 8, A, A, 4, 128, None) == -3
    assert lib.plx_kv_quantize_fp8(A, A, A + 2, 4, 128, None) == -3      # scales need 4 bytes
    # plx_decode_fp8kv(q, r, Kc, Ks, Vc, Vs, seqlens, out, B, H, Hkv, L, d, ws, ws_bytes, stream)
    ok = [A] * 8
    assert lib.plx_decode_fp8kv(A, A, A, None, A, A, A, A, 1, 8, 2, 64, 128, None, 0, None) == -1
    assert lib.plx_decode_fp8kv(*ok, 1, 8, 3, 64, 128, None, 0, None) == -1   # H not a multiple of Hkv
    assert lib.plx_decode_fp8kv(*ok, 1, 6, 2, 64, 128, None, 0, None) == -2   # group of 3
    assert lib.plx_decode_fp8kv(*ok, 1, 32, 2, 64, 128, None, 0, None) == -2  # group of 16
    assert lib.plx_decode_fp8kv(*ok, 1, 8, 2, 64, 64, None, 0, None) == -2    # d = 128 only
    assert lib.plx_decode_fp8kv(A + 4, A, A, A, A, A, A, A, 1, 8, 2, 64, 128, None, 0, None) == -3
    assert lib.plx_decode_fp8kv(A, A, A, A + 4, A, A, A, A, 1, 8, 2, 64, 128, None, 0, None) == -3  # scales 16 B
    assert lib.plx_decode_fp8kv(A, A, A, A, A, A, A + 2, A, 1, 8, 2, 64, 128, None, 0, None) == -3  # seqlens 4 B
    assert lib.plx_decode_fp8kv(*ok, 1 << 22, 8, 8, 64, 128, None, 0, None) == -2  # B*H above 2^24
    assert lib.plx_decode_fp8kv_workspace_bytes(1, 8, 3, 64, 128) == 0
    S = lib.plx_decode_num_splits(1, 2, 8192, 128)
    assert S > 1 and lib.plx_decode_fp8kv_workspace_bytes(1, 8, 2, 8192, 128) == 8 * S * (2 * 128 + 4) * 4


def test_dilated_prefill_rejects_bad_arguments(lib):
    # plx_prefill_dilated(Q, K, V, R, out, B, H, Hkv, N, d, dilation, window, stream)
    ok = [A] * 5
    assert lib.plx_prefill_dilated(None, A, A, A, A, 1, 4, 2, 256, 128, 2, 0, None) == -1
    assert lib.plx_prefill_dilated(*ok, 1, 4, 2, 256, 128, 0, 0, None) == -1      # dilation >= 1
    assert lib.plx_prefill_dilated(*ok, 1, 4, 2, 256, 128, 2, -1, None) == -1     # window >= 0
    assert lib.plx_prefill_dilated(*ok, 1, 4, 3, 256, 128, 2, 0, None) == -1      # H not a multiple of Hkv
    assert lib.plx_prefill_dilated(*ok, 1, 4, 2, 300, 128, 7, 0, None) == -2      # ragged classes
    assert lib.plx_prefill_dilated(*ok, 1, 4, 2, 256, 96, 2, 0, None) == -2
    assert lib.plx_prefill_dilated(A, A, A + 8, A, A, 1, 4, 2, 256, 128, 2, 0, None) == -3
    assert lib.plx_prefill_dilated(*ok, 1 << 20, 16, 16, 256, 128, 2, 0, None) == -2  # B*H*r above 2^24


def test_layer_and_norm_rope_reject_bad_arguments(lib):
    assert lib.plx_qkr_norm_rope(None, A, 1, 8, 2, 128, 1e-6, 1e4, None) == -1
    assert lib.plx_qkr_norm_rope(A, A, 1, 8, 2, 96, 1e-6, 1e4, None) == -2
    assert lib.plx_qkr_norm_rope(A, A, 1, 8, 2, 128, -1.0, 1e4, None) == -1
    assert lib.plx_layer_forward(*([A] * 6), None, 1, 8, 2, 128, None, 0, None) == -1
    assert lib.plx_layer_forward(*([A] * 7), 1, 8, 2, 32, None, 0, None) == -2
    assert lib.plx_layer_forward(*([A] * 6), A + 4, 1, 8, 2, 128, None, 0, None) == -3


def test_decode_split_plan(lib):
    # Sizes on both sides of the kernel choice (tensor-core decode: one CTA
    # per SM; warp-MMA decode: two), whose split plans differ.
    for (B, H, L) in [(64, 16, 4096), (1, 16, 32768), (2048, 16, 4096), (1, 1, 1), (3, 5, 1000),
                      (1, 16, 128), (8, 16, 16384), (64, 16, 1024), (256, 16, 1024), (16, 16, 2048),
                      (8, 16, 2048), (1, 16, 16384), (3, 7, 20000)]:
        S = lib.plx_decode_num_splits(B, H, L, 128)
        assert 1 <= S <= max(1, L // 256) + 1
        ws = lib.plx_decode_workspace_bytes(B, H, L, 128)
        if S == 1:
            assert ws == 0
        else:
            assert ws == B * H * S * (2 * 128 + 4) * 4
    # Small batches split the context; large ones do not need to.
    assert lib.plx_decode_num_splits(1, 16, 32768, 128) > 8
    assert lib.plx_decode_num_splits(2048, 16, 4096, 128) == 1


def test_layer_workspace_slots_match_the_binding():
    """The caller workspace of plx_layer_forward holds nine 256-byte-aligned
    slots; the binding's views of the layer's own attention inputs and output
    are slots 4..8, [B, H, N, d] bf16 each."""
    import torch
    from local_linear_attention_streamed_b200 import plx
    for (B, N, H, d) in [(1, 1, 1, 64), (2, 100, 3, 64), (4, 8192, 16, 128), (3, 7, 5, 128)]:
        slot = -(-(B * N * H * d * 2) // 256) * 256
        assert plx.layer_workspace_bytes(B, N, H, d) == 9 * slot
        if B * N * H * d > 1 << 20:
            continue
        ws = torch.zeros(9 * slot, dtype=torch.uint8)
        views = plx.layer_workspace_views(ws, B, N, H, d)
        base = ws.data_ptr()
        for i, name in enumerate(("q", "k", "v", "rho", "attn")):
            t = views[name]
            assert t.dtype == torch.bfloat16 and tuple(t.shape) == (B, H, N, d)
            assert t.data_ptr() - base == (4 + i) * slot
