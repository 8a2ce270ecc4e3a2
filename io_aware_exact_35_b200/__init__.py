"""B200-native exact IO-aware attention: forward, recomputing backward and
split-KV decode, behind the C-ABI library ``libfa_b200.so``.

Importing the package loads nothing; ``io_aware_exact_35_b200.fa`` loads the
compiled library on first use and raises if it is missing.
"""
__all__ = ["fa", "inputs", "autograd"]
