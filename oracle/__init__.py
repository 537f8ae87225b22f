"""Float64 CPU oracle of the flash-CCE ORPO head (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs may import this package.  It shares no code with the CUDA library.
"""
from .flash_cce import *  # noqa: F401,F403
