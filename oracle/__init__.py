"""CPU fp64 oracle of the Sign-Muon step (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs may import this package.  The CUDA product path never does.
"""
from .signmuon_oracle import *  # noqa: F401,F403
from .signmuon_oracle import NS_QUINTIC, NORM_EPS  # noqa: F401
