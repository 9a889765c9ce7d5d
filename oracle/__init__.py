"""CPU oracle for the SSTA forward pass (test infrastructure only).

Only tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  The CUDA library never does, and this package never
imports the CUDA library.
"""
from .ssta_oracle import *  # noqa: F401,F403
from .ssta_oracle import __all__  # noqa: F401
