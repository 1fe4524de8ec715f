"""Float64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
baseline leg of the benchmark may import this package.  The library's
product path never calls it and has no CPU fallback.
"""

from .attention import (  # noqa: F401
    diag_offset,
    visible_mask,
    visible_band,
    attention_weights,
    attn_fwd,
    attn_fwd_rows,
    attn_bwd,
    attn_row_block,
)
