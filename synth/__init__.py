"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This package only draws random inputs (pair tables, angles, scales, weights,
activations).  It holds none of the method's arithmetic: no rotation, fold,
quantisation, packing or matmul lives here.
"""
from .inputs import (  # noqa: F401
    LAYER_SHAPES,
    LinearProblem,
    bf16_round,
    config_problems,
    device_weights,
    linear_problem,
)
