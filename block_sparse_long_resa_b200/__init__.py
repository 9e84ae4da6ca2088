"""B200-native hot path of Rectified Sparse Attention (ReSA).

The compute lives in ``libresa.so`` (hand-written CUDA for sm_100a behind a
C ABI declared in include/resa.h); ``block_sparse_long_resa_b200.resa`` is the
thin ctypes binding.  Importing this package does not load the library; the
binding does, and fails loudly when it is missing.
"""
__all__ = ["inputs", "resa"]
