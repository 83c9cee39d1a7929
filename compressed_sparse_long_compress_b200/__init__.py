"""B200-native hybrid compressed attention (CSA + HCA) for sm_100a.

The compute path is the C-ABI library ``libcslc.so`` (CUDA kernels under
``csrc/``, declared in ``include/cslc.h``); ``cslc`` is its Python binding.
"""

__all__ = ["cslc", "workloads"]
