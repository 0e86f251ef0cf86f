"""B200-native routed-MoE layer (MLX affine 4-bit experts, 8-bit router).

The compute lives in libmoe.so (hand-written CUDA for sm_100a); this package
is its thin Python binding plus device-memory plumbing.  Importing it loads
the library and fails loudly if it has not been built.
"""
from ._lib import MoeError, lib  # noqa: F401
from .binding import *  # noqa: F401,F403

lib()
