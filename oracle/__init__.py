"""fp64 CPU oracle of the fused chunked top-K KL loss and of the teacher
top-K cache writer (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  The product library never
does, and the two share no code.
"""

from .kd_oracle import *  # noqa: F401,F403
from .kd_oracle import __all__ as _kd_all
from .topk_cache import teacher_topk  # noqa: F401

__all__ = list(_kd_all) + ["teacher_topk"]
