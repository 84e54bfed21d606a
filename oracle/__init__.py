"""fp64 CPU oracle of the Medusa verification step.

TEST INFRASTRUCTURE: imported only by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``.  The CUDA library never imports it.
"""

from .medusa_oracle import *  # noqa: F401,F403
