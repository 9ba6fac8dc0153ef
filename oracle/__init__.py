"""CPU float64 oracle for CLEAR attention. Test infrastructure only: imported by tests/,
__graft_entry__.smoke() and bench.py's CPU-baseline / reference legs, never by the product path."""
from .clear_attention import (  # noqa: F401
    WINDOWS,
    token_coords,
    window_half_width,
    clear_mask,
    clear_attention_forward,
    clear_attention_rows,
    clear_attention_backward,
    window_lattice_count,
    window_pairs,
    kept_pairs,
    useful_flops_fwd,
    clear_attention_stripe,
    clear_text_rows_patch_average,
    e4m3_decode,
    clear_attention_forward_fp8,
)
