"""fp64 CPU oracle for exact attention: test infrastructure, never the product path.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs import this package.
"""
from .attention import *  # noqa: F401,F403
from .attention import __all__  # noqa: F401
