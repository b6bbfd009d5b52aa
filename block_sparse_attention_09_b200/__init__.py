"""B200-native MiniMax Sparse Attention (MSA) training hot path.

The compute lives in ``libmsa.so`` (hand-written CUDA for sm_100a behind a C
ABI declared in ``include/msa.h``); ``msa`` is its thin ctypes binding and
``inputs`` the seeded synthetic-input recipes.  Import ``msa`` explicitly:
importing the package itself loads nothing.
"""
__all__ = ["inputs", "msa"]
