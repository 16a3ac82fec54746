"""CPU oracle of the ternary weight path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  It shares no code with the CUDA library.
"""
from .oracle import *  # noqa: F401,F403
from .oracle import build  # noqa: F401
