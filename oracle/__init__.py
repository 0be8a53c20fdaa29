"""CPU oracle for the partial-recompute denoising step (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and the
product path has no CPU fallback.
"""
from .plk_oracle import *  # noqa: F401,F403
