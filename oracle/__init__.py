"""fp64 CPU oracle for RMSNorm fused into its linear projection (FlashNorm form).

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline
leg of the benchmark may import this package.  The library never calls it and
shares no code with it: the CUDA path lives in the
``rmsnorm_linear_projection_flashnorm_b200`` package and neither imports the
other.  Both take their inputs from the ``workloads`` generators, which hold
none of the method's arithmetic.

Every function here is pinned by a CPU test against something other than
itself (closed forms, invariants, brute force, torch's own casts); see
``tests/test_oracle.py``.
"""
from .flashnorm_oracle import *  # noqa: F401,F403
