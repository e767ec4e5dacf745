"""CPU oracle for the FP8 grouped matmul (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding in ``moe_fp8_grouped_b200``) never imports it.
"""
from .oracle import *  # noqa: F401,F403
