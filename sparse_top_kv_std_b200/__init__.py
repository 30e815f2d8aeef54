"""Sparse-to-Dense (StD) decoding hot path for B200 (sm_100a).

The compute lives in ``libstd_b200.so`` (hand-written CUDA kernels behind the C
ABI of include/std_b200.h); ``binding`` exposes its entry points to Python
with the same names.  The library is loaded on first use, and a missing
library raises instead of falling back to anything else.
"""
from . import binding  # noqa: F401
from .binding import StdError, dims, lib  # noqa: F401

__all__ = ["binding", "StdError", "dims", "lib"]
