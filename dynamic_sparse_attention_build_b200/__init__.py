"""B200-native dynamic sparse attention for long-context prefill.

Two calls, implemented as sm_100a CUDA kernels in ``libdsa.so`` (C ABI in
``include/dsa.h``):

* ``build_indices(Q, K, patterns, block)``: per-head sparse indices (A-shape,
  Vertical-Slash, block top-k, block threshold, MoBA routing);
* ``sparse_prefill(Q, K, V, indices)``: causal block-sparse attention over the
  selected key blocks and columns.

Importing the package does not load the library; the first call does, and fails
loudly if it has not been built (``python -m dynamic_sparse_attention_build_b200.build``).
"""
from .api import (HostPrefill, IndexBuffers, alloc_indices, build_indices, count_pairs,  # noqa: F401
                  device_status, indices_from_lists, make_patterns, make_problem, sparse_prefill)
