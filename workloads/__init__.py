"""Seeded synthetic inputs for block-sparse variable-length attention.

This package only draws random numbers and lays them out in the tensor
shapes the operator takes (Q/K/V/dOut, the uint16 block index, cu_seqlens,
seqused_kv, the paged block table). It contains none of the attention
arithmetic, so both the CPU oracle and the CUDA path can take their inputs
from here without sharing any of the method's code.
"""
from .gen import Problem, CONFIGS, make_config, make_problem, NO_BLOCK  # noqa: F401
