"""CPU oracle for the S3R per-round hot path (test infrastructure, not product code).

Only the test suite, the smoke check in ``__graft_entry__`` and the CPU-baseline /
reference legs of ``bench.py`` may import this package. The CUDA library never calls it,
and it shares no code with the CUDA path.
"""
from .s3r_oracle import *  # noqa: F401,F403
