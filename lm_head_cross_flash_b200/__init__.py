"""flash-CCE ORPO language-model head for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libcce.so`` (hand-written CUDA for
sm_100a) declared in ``include/cce.h``; ``lm_head_cross_flash_b200.cce`` is a
thin ctypes binding with the same entry-point names.  Importing this package
does not load the library; the first call does, and raises if it is missing.
"""

__all__ = ["cce", "synthetic"]
