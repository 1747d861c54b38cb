"""Seeded synthetic inputs for the sparse MoE FFN layer.

This package holds only input generation: shapes, random draws and the
offline FP8 encoding of expert weights (the layer consumes FP8 weights as
given inputs).  It contains none of the layer's own arithmetic, and both the
CPU oracle and the CUDA library are fed from it.
"""
from .inputs import (  # noqa: F401
    MoEShape,
    WORKLOADS,
    DTYPE_F32,
    DTYPE_BF16,
    DTYPE_FP8,
    make_inputs,
    encode_fp8_blocks,
)
