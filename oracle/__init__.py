"""fp64 CPU oracle for the sparse top-k MoE layer.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg use it.  The CUDA library never imports, links or calls it.
"""

from .oracle import *  # noqa: F401,F403
