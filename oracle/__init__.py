"""fp64 CPU oracle for chunkwise GLA / GSA and the elementwise pieces around them.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference legs, never by the library package.
"""
from .gla_oracle import *  # noqa: F401,F403
from .gla_oracle import __all__ as _gla_all
from .aux_oracle import *  # noqa: F401,F403
from .aux_oracle import __all__ as _aux_all

__all__ = list(_gla_all) + list(_aux_all)
