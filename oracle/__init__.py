"""fp64 CPU oracle for the Muon optimizer step (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import this package. The CUDA library never does.
"""

from .muon_oracle import *  # noqa: F401,F403
from .muon_oracle import StepParams, FlopCounter  # noqa: F401
