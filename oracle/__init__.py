"""Plain CPU oracle of the ParoQuant runtime hot path.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
bench's CPU-baseline leg may import this package.  The CUDA library never
calls into it and shares no code with it.
"""
from .paro import (  # noqa: F401
    dequantize,
    fold_weights,
    givens_stage,
    linear,
    pack_nibbles,
    quantize_groups,
    rotate,
    rotate_w4_linear,
    unpack_nibbles,
    w4_linear,
    pack_weights,
    check_stage_disjoint,
)
from .backward import rotate_backward  # noqa: F401,E402
from .w4a4 import dequantize_activations, quantize_activations, rotate_w4a4_linear, w4a4_linear  # noqa: F401,E402
