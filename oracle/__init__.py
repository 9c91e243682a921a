"""CPU oracle for block-sparse attention prefill -- TEST INFRASTRUCTURE ONLY.

A plain float64 restatement of what the method computes (pooling, scoring,
selection, masked attention), used to check the CUDA library.  Only the test
suite, the package entry file's smoke check and the benchmark's CPU-baseline
and reference legs may import it.  The library never imports it and shares no
code with it; the only common module is the seeded workload generator.
"""
from .sbsa_oracle import *  # noqa: F401,F403
