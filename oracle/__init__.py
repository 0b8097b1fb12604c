"""CPU fp64 oracle for the large-chunk TTT layer.

TEST INFRASTRUCTURE ONLY: imported by the test suite, by the package smoke
check and by the bench's CPU-baseline / reference legs, never by the product
path.  It shares no code with the CUDA library.
"""
from .ttt_oracle import *  # noqa: F401,F403
