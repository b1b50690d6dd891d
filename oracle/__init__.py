"""fp64 CPU oracle of the SparsePR attention call (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference arm
may import this package; the CUDA library never does.
"""
from . import sparsepr_oracle  # noqa: F401
