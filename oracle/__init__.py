"""fp64 CPU oracle of the BPT layer forward (and its gradients).

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
from .bpt_oracle_backward import (  # noqa: F401
    attention_backward,
    attention_backward_blockwise,
    layer_backward,
)
