"""Float64 CPU oracle of the selective scan (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA library does not depend on it.
"""
from .oracle import (BBAR_DELTA, BBAR_ZOH, LIBRARY, SOURCE, Oracle, build,
                     default, default_threads)

__all__ = ["Oracle", "build", "default", "default_threads", "BBAR_DELTA",
           "BBAR_ZOH", "LIBRARY", "SOURCE"]
