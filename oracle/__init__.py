"""CPU oracle for the SPADE executor hot path (test infrastructure only).

Only the tests, the smoke check in __graft_entry__ and the CPU-baseline leg of
bench.py may import this package.  The library never calls it.
"""
from .spade_oracle import *  # noqa: F401,F403
