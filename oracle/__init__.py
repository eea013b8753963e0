"""fp64 CPU oracle of the AuraFlow denoising forward (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The CUDA library never calls it and shares no
code with it.
"""
from .auraflow import *  # noqa: F401,F403
