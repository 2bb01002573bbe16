"""fp64 CPU oracle for the ISPA hot path -- test infrastructure only.

Imported by tests/, by __graft_entry__.smoke() and by the CPU-baseline leg of
bench.py.  Never imported by the product package or its CUDA library.
"""
from .ispa_oracle import *  # noqa: F401,F403
from . import ispa_oracle  # noqa: F401
