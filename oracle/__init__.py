"""CPU oracle for SharQ's sparse-dense FP4 linear layer.

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and bench.py's CPU
baseline may import it; the product path (the CUDA library and its binding) never does.
"""
from . import formats, layouts, sharq  # noqa: F401
