"""CPU oracle for the chunk-wise Gated DeltaNet inversion + WY path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use it.  It shares no code with the CUDA library and imports
nothing from it.

Everything here is plain numpy, float64 unless a function states otherwise
(the INT8 scheme is integer + IEEE float32 by construction).  See
``oracle/gdn_oracle.py`` for the functions and the passages each follows.
"""
from .gdn_oracle import *  # noqa: F401,F403
