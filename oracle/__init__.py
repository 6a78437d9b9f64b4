"""fp64 CPU oracle of the BPT layer forward.

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the
benchmark's CPU-baseline leg use it to produce expected values. The library
never imports it, and it imports nothing from the library.
"""

from .bpt_oracle import (  # noqa: F401
    attention,
    attention_blockwise,
    layer_forward,
    layer_forward_blockwise,
    layer_rows,
    qkv_projection,
    residual_ffn,
)
