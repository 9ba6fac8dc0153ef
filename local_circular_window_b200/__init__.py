"""B200-native CLEAR attention (circular local window + global text tokens), forward and backward.

Compute runs in libclear_attn.so (hand-written sm_100a kernels behind a C ABI, see
include/clear_attn.h); this package only marshals arguments. The binding is imported lazily so
that ``python -m local_circular_window_b200.build`` works before the library exists; any other
attribute access loads it and raises ImportError if it was never built.
"""
import importlib

_EXPORTS = {
    "CLEAR_OK", "ClearError", "ClearParams", "LIB_PATH", "bwd_workspace_size", "clear_attn_bwd",
    "clear_attn_check", "clear_attn_fwd", "clear_attn_fwd_host", "clear_attn_fwd_strided", "ClearStrides",
    "device_diag", "forward_shape", "ClearStripe", "make_stripe", "clear_attn_fwd_stripe", "clear_attn_text_merge",
    "fwd_host_workspace_size", "fwd_workspace_size", "header_functions", "item_tiles", "lib", "make_params",
    "pair_counts", "selftest_expiry", "status_string", "version", "clear_attn_fwd_varlen", "varlen_workspace_size",
    "varlen_tokens", "clear_attn_fwd_fp8", "clear_attn_fwd_rope", "rope_workspace_size", "ClearRope",
    "clear_attn_rope", "rope_rotate_workspace_size", "clear_attn_bwd_rope",
}


def __getattr__(name):
    if name in _EXPORTS:
        return getattr(importlib.import_module("._binding", __name__), name)
    raise AttributeError(name)


def __dir__():
    return sorted(_EXPORTS)
