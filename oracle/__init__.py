"""fp64 CPU oracle of the fused chunked top-K KL loss (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  The product library never
does, and the two share no code.
"""

from .kd_oracle import *  # noqa: F401,F403
from .kd_oracle import __all__  # noqa: F401
