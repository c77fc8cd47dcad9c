"""MISA token indexer on B200 (sm_100a): a C-ABI library of hand-written CUDA
kernels (libmisa.so) and a thin Python binding.

Importing the package does not touch the GPU; importing `ops` (the binding)
loads libmisa.so and fails loudly when it has not been built.
"""
from . import workloads  # noqa: F401

__all__ = ["workloads"]


def ops():
    """The C-ABI binding module (loads libmisa.so)."""
    from . import _lib
    return _lib
