"""CPU oracle for the Sparse Query Attention hot path (test infrastructure).

This package is a plain, slow, fp64 restatement of what the attention core,
its gradient and the reduced-width projections compute.  It exists to check
the CUDA path and shares no code with it.  Only the test suite, the smoke
check and the benchmark's CPU-baseline leg may import it; the product never
does.
"""

from .sqa_oracle import (  # noqa: F401
    attention_forward,
    attention_backward,
    attention_decode,
    projection,
    projection_backward,
    sqa_layer_backward,
    sqa_layer_forward,
)
