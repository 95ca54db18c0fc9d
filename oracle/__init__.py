"""Float64 CPU oracle for CSA + HCA compressed attention.

Test infrastructure only: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline legs of ``bench.py``; never by the product path.
"""

from .csahca_oracle import *  # noqa: F401,F403
from . import csahca_oracle  # noqa: F401
