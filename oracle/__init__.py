"""Float64 CPU oracle for CCGQA (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package.  It shares no code with the CUDA path and
imports nothing from the product package.  See ``oracle/ccgqa.py``.
"""
from . import ccgqa  # noqa: F401
