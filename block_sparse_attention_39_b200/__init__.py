"""PBSA (Persistent Block-Sparse Attention) hot path for NVIDIA B200 (sm_100a).

The compute lives in the C-ABI library ``libpbsa.so`` (``include/pbsa.h``);
``pbsa`` is its Python binding (same names), ``engine`` keeps one layer's
device state and runs the chunk step through the ABI.
"""
from . import pbsa  # noqa: F401
from ._lib import LIB_PATH, lib  # noqa: F401

__all__ = ["pbsa", "lib", "LIB_PATH"]
