"""Independent CPU oracle of the MISA / DSA indexer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA
library under ``long_context_misa_b200/``.
"""
from . import misa_oracle  # noqa: F401
