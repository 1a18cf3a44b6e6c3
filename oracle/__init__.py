"""CPU oracle for the sparse-attention decode path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  The CUDA library never calls it, and it never calls the
CUDA library: the two share no code.
"""
from .ls_oracle import *  # noqa: F401,F403
