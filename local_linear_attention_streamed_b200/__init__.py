"""Parallax attention on B200: C-ABI library (libplx.so) plus a thin Python binding.

The binding is loaded on first use of a compute entry point; importing this
package alone (for example, to reach the seeded input generator in ``synth``)
does not need the compiled library.  Every compute call goes through
``libplx.so``; if it is missing the call raises instead of falling back.
"""

_BINDING_NAMES = {
    "prefill", "decode", "decode_gqa", "decode_noalloc", "decode_workspace_bytes", "layer_forward", "qkr_norm_rope",
    "get_device_status", "status_string", "PlxError", "lib", "PLX_F32", "PLX_BF16",
    "prefill_train", "prefill_backward", "prefill_bwd_workspace_bytes", "parallax_attention",
    "ParallaxAttention", "prefill_window", "decode_window", "layer_forward_fp8", "prefill_block_sparse", "prefill_gqa",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import plx
        return getattr(plx, name)
    raise AttributeError(name)
