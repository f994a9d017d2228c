"""Float64 CPU oracle for Parallax attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The CUDA library never calls it, and it never
calls the CUDA library.
"""
from .parallax import (decode_gqa_ref, decode_ref, parallax_row, prefill_block_sparse_ref, prefill_dilated_ref,
                       prefill_gqa_ref, prefill_ref, softmax_weights_row)
from .layer import (e4m3, fp8_linear, fp8_per_tensor, layer_fp8_ref, layer_rows_ref, qkr_norm_rope_ref, rmsnorm,
                    rope)
from .backward import parallax_backward_ref, parallax_forward_ref, prefill_stats_ref
from .lla import lla_prefill_ref, lla_probe, lla_row
from .kvfp8 import decode_fp8kv_ref, e4m3_bits, e4m3_value, kv_dequantize_fp8_ref, kv_quantize_fp8_ref

__all__ = ["parallax_row", "prefill_ref", "prefill_block_sparse_ref", "prefill_dilated_ref", "prefill_gqa_ref", "decode_ref", "decode_gqa_ref", "softmax_weights_row",
           "layer_rows_ref", "qkr_norm_rope_ref", "rmsnorm", "rope",
           "e4m3", "fp8_linear", "fp8_per_tensor", "layer_fp8_ref",
           "parallax_backward_ref", "parallax_forward_ref", "prefill_stats_ref",
           "lla_prefill_ref", "lla_probe", "lla_row",
           "decode_fp8kv_ref", "e4m3_bits", "e4m3_value", "kv_dequantize_fp8_ref", "kv_quantize_fp8_ref"]
