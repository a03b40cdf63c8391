"""fp64 CPU oracle for the DoRA hot path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  The product library never does.
"""
from .dora_oracle import *  # noqa: F401,F403
from .dora_oracle import __all__  # noqa: F401
