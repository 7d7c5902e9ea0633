"""CPU oracle of the ConvRot W4A4 linear -- test infrastructure only.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It shares no code with the CUDA library.
"""
from .oracle import *  # noqa: F401,F403
