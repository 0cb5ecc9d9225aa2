"""fp64 CPU oracle of the block-sparse video attention forward.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py``; never by the library itself. It shares
no code with the CUDA path.

Every function is pinned by the CPU tests in ``tests/test_oracle_pins.py`` (closed
forms, library special cases, invariants and hand-derived fixtures).
"""
from .spark_oracle import *  # noqa: F401,F403
