"""CPU oracle for the 1-bit group-128 hot path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference legs may import this package.  It shares no code with the CUDA
library and never imports it.
"""
from .w1_oracle import *  # noqa: F401,F403
