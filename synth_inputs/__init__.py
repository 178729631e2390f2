"""Seeded synthetic layers for two-sided GPTQ: weights W and Kronecker factors A, B.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark, so that both sides read the same bytes.  It contains none of the
quantization method's arithmetic: no damping, no factorization, no scales, no
rounding.  It only draws random numbers and forms the calibration statistics
A = X^T X / N and B = G^T G / N that a caller would otherwise accumulate from
activations X and output gradients G.

The recipe follows the synthetic Llama-3-8B-class layers described for the
two-sided GPTQ workloads (FastKron / BaKron page, Section 2.7 and Table 3, where
only the shapes and the 14336x4096 / 4096x4096 sizes survive).
"""
from .layers import (  # noqa: F401
    LayerSpec,
    WORKLOADS,
    layer_inputs,
    workload,
)
