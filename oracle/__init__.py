"""CPU oracle for the grouped 4-bit MoE GEMM -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The library never does.
"""
from . import gnf4_oracle  # noqa: F401
from . import storage  # noqa: F401
