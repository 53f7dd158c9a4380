"""FP64 CPU oracle for LLA decode attention — test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs may import this package.  It shares no code with the CUDA library.
"""

from . import bruteforce, lla_oracle  # noqa: F401
