"""CPU oracles for the hybrid compressed attention path (test infrastructure).

Two independent float64 restatements of the method: ``cslc_oracle`` (numpy,
re-exported here) and ``cpp_oracle`` (a C++ / OpenMP library behind the same
Python API). Both are pinned by the same tests. Only the test suite,
``__graft_entry__.smoke()`` and the CPU-baseline legs of ``bench.py`` may import
this package. The product path never does: the CUDA library under
``compressed_sparse_long_compress_b200`` shares no code with either.
"""

from .cslc_oracle import *  # noqa: F401,F403
