"""CPU oracle of the VSA forward path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA
library and never loads it.
"""
from . import vsa_oracle  # noqa: F401
