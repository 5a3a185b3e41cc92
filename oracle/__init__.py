"""fp64 CPU oracle for the DSA hot path.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline leg of bench.py, never by the library.  See dsa_oracle.py.
"""
from .dsa_oracle import *  # noqa: F401,F403
