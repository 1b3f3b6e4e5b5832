"""fp64 CPU oracle of the large-chunk TTT layer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this package.  The CUDA product path never does.
"""
from .ttt_oracle import *  # noqa: F401,F403
from .ttt_oracle import RENORM_FROB, RENORM_OFF, RENORM_ROW  # noqa: F401
