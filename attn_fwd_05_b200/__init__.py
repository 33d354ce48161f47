"""Exact attention for one NVIDIA B200 (sm_100a) behind a small C ABI.

The CUDA library (``libattn_b200.so``, built from ``csrc/``) does all the
work; this package only marshals torch tensors into its entry points.  The
library is loaded on first use and a missing or unloadable library raises
``RuntimeError``: there is no CPU fallback.
"""

from .binding import (  # noqa: F401
    AttnError,
    attn_bwd,
    attn_bwd_workspace_size,
    attn_decode_paged,
    attn_decode_paged_noalloc,
    attn_decode_paged_workspace_size,
    attn_fwd,
    attn_fwd_ex,
    attn_fwd_fp8,
    attn_fwd_masked,
    attn_get_device_status,
    attn_quantize_fp8,
    attn_debug_bwd_stall,
    attn_debug_decode_stall,
    attn_debug_exp2,
    attn_debug_fwd_stall,
    attn_debug_watchdog,
    attn_status_string,
    library_path,
    load_library,
)
