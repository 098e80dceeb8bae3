"""B200-native GQA-adapted DeepSeek Sparse Attention (DSA) layer.

The compute path is the CUDA library ``libdsa.so`` (sm_100a kernels behind a
C ABI declared in ``include/dsa.h``); ``sparse_long_context_03_b200.dsa`` is
its thin ctypes binding.  ``inputs`` holds the seeded synthetic workloads.
Importing this package loads nothing: the library is opened on first use and
a missing library raises instead of falling back to anything else.
"""
__all__ = ["dsa", "inputs"]
