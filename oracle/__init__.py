"""CPU float64 oracle for the VDN hybrid attention forward.

Test infrastructure only: imported by the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product path.
"""
from . import vdn_oracle  # noqa: F401
