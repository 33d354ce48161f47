"""fp64 CPU oracle for exact attention, its gradients and paged-KV decode.

Test infrastructure: used only by the tests, the smoke check and the
benchmark's CPU-baseline leg.  It shares no code with the CUDA library.
"""

from .attention import (  # noqa: F401
    as_f64,
    attention,
    attention_head,
    attention_rows,
    causal_visible,
    decode_paged,
    gather_pages,
    kv_head_of,
    visible_mask,
)
from .backward import attention_backward, attention_head_backward  # noqa: F401
from .fp8 import attention_fp8_reference, block_quantize, dequantize, e4m3_value, quantize_e4m3  # noqa: F401
