"""fp64 CPU oracle for FAVOR+ attention.

TEST INFRASTRUCTURE: imported only by tests/, by __graft_entry__.smoke() and
by bench.py's cpu_baseline and reference legs.  It shares no code with the
CUDA library, and the library never imports it.
"""
from . import philox, favor  # noqa: F401
