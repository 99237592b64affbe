"""B200 (sm_100a) Native Sparse Attention / MoBA forward library.

The compute lives in ``libnsa_b200.so`` (C ABI in ``include/nsa.h``); the
binding is :mod:`dynamic_block_sparse_nsa_b200.nsa`. Importing the package
itself loads nothing, so the input generators can be used without a GPU.
"""
