"""fp64 CPU oracle for the OrbitQuant online quantized-linear path.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this package.
The product library never imports it and shares no code with it.

Functions whose result is not pinned to something outside the oracle: none.  Every entry
point is checked in ``tests/test_oracle_*.py`` against published values, closed forms,
invariants, brute force or an independent library computation (see each test's docstring).
"""
from .oracle import *  # noqa: F401,F403
