"""fp64 CPU oracle of Gated MLA: test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
and reference legs import this package. The CUDA library never does.
"""
from .gmla_oracle import *  # noqa: F401,F403
from . import gmla_oracle as core  # noqa: F401
