"""CPU oracle for the hybrid compressed attention path (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path never does: the CUDA
library under ``compressed_sparse_long_compress_b200`` shares no code with it.
"""

from .cslc_oracle import *  # noqa: F401,F403
