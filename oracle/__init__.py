"""fp64 CPU oracle for the VGGT attention path -- test infrastructure only.

Imported by ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline; never by the product path.
"""
from . import vggt_oracle  # noqa: F401
