"""CPU oracle for the MoE layer hot path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The library never does: its product
path runs only in the CUDA kernels of ``libmoe``.
"""
from . import oracle  # noqa: F401
