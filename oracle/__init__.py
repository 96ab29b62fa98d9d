"""Plain float64 CPU oracle for the Prefix Sliding attention hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this package.  The CUDA
library never calls it and shares no code with it.
"""
from .ps_oracle import *  # noqa: F401,F403
from .ps_oracle import __all__  # noqa: F401
