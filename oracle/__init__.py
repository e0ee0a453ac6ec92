"""CPU oracle for the IndexCache hot path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline
may import this package.  It shares no code with the CUDA library.
"""
from .indexcache_oracle import *  # noqa: F401,F403
from .indexcache_oracle import __all__  # noqa: F401
