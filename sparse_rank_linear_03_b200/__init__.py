"""B200-native S + U Vᵀ compressed linear layers (hierarchical sparse + low-rank).

The compute path lives in ``libhsl.so`` (CUDA for sm_100a behind a C ABI,
declared in ``include/hsl.h``); ``sparse_rank_linear_03_b200.hsl`` is the
ctypes binding.  Importing this package does not load the library; importing
``.hsl`` does, and fails loudly if it has not been built.
"""
__version__ = "0.1.0"
