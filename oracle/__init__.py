"""fp64 CPU oracle for chunkwise GLA / GSA.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference legs, never by the library package.
"""
from .gla_oracle import *  # noqa: F401,F403
from .gla_oracle import __all__  # noqa: F401
