"""CPU oracle (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  It shares no code with the CUDA path and the library never
calls it.  See ``fp4q_oracle`` for the definitions and their sources.
"""

from .fp4q_oracle import *  # noqa: F401,F403
from .fp4q_oracle import (E2M1_MAGNITUDES, E2M1_MIDPOINTS, E4M3_MAX,  # noqa: F401
                          NV_TENSOR_DIVISOR)
