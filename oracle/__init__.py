"""fp64 CPU oracle of the routed-MoE layer and the LFU slot-cache simulator.

TEST INFRASTRUCTURE: only the tests, the package smoke check and the
benchmark's CPU-baseline leg may import anything here.  It shares no code
with the CUDA library and imports nothing from it.
"""
from . import moe_oracle, lfu_sim  # noqa: F401
