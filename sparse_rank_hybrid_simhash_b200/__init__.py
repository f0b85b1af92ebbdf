"""B200-native ELSAA attention (libelsaa): SimHash + Sort-LSH exact sparse branch,
RACE low-rank branch, denominator-aware fusion and token-wise gates, forward
and backward, as hand-written sm_100a CUDA kernels behind a C ABI.

Importing the package loads nothing; the first call into ``binding`` loads
``libelsaa.so`` and raises if it is missing.
"""

from . import workloads  # noqa: F401

__all__ = ["binding", "workloads"]
