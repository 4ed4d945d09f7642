"""CPU oracle for COBS block-sparse decode — test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never does.
"""

from .cobs_oracle import *  # noqa: F401,F403
from .cobs_oracle import __all__  # noqa: F401
