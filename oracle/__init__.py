"""CPU oracle for the routed low-bit MoE layer -- TEST INFRASTRUCTURE ONLY.

Plain, slow, fp64 NumPy restatement of what the layer computes.  It shares no
code with the CUDA library and must never be imported by the product path:
only the test-suite, the smoke check and the benchmark's CPU-baseline leg use
it.
"""
from .moe_oracle import *  # noqa: F401,F403
