"""Seeded synthetic inputs for the routed-MoE layer (weights, biases, rows).

This package draws random numbers and lays bytes out; it holds none of the
layer's arithmetic (no dequantisation, no matmul, no routing).  Both the
fp64 oracle and the CUDA path read what it produces.
"""
from .synth import *  # noqa: F401,F403
from .configs import CONFIGS, Config, tiny_config  # noqa: F401
