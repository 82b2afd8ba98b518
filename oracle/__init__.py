"""fp64 CPU oracle for blockwise exact ("ring") attention.

Test infrastructure only: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline legs of ``bench.py``; never by the library.
"""
from .ring_oracle import *  # noqa: F401,F403
from .ring_oracle import __all__  # noqa: F401
