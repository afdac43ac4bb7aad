"""CPU fp64 oracle for dynamic sparse attention prefill.

Test infrastructure only: imported by ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference legs of ``bench.py``.  Never by the product package.
"""
from .dsa_oracle import *  # noqa: F401,F403
