"""Seeded synthetic inputs for HiLS-Attention.

This module only draws random tensors and lays them out; it holds none of the
method's arithmetic.  Both the fp64 oracle (through the tests) and the CUDA
path consume what it returns.
"""
from .generate import (  # noqa: F401
    PrefillInputs,
    DecodeInputs,
    prefill_inputs,
    decode_inputs,
    CONFIGS,
)
