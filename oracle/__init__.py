"""CPU oracle for the Q4_K weight-only matrix products -- test infrastructure.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library
under ``q4_weight_only_super_b200/`` and its binding) never imports, links or
runs anything here, and the two share no code.
"""
from . import q4k  # noqa: F401
