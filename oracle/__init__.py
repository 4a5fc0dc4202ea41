"""CPU oracle for token-sparse decode attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls it, and shares no code with
it: the two meet only at the seeded inputs drawn by ``dsgen``.

``oracle.cxx`` is the C++ oracle (ds_oracle.cpp) with the same function names
and results; it shares no code with the numpy oracle below.
"""
from .ds_oracle import *  # noqa: F401,F403
