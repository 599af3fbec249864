"""MSA (MiniMax Sparse Attention) hot path for B200 (sm_100a).

The compute lives in a C-ABI shared library built from ``csrc/`` (declared in
``include/msa.h``); :mod:`block_sparse_long_scores_b200.msa` is its thin ctypes binding and
:mod:`block_sparse_long_scores_b200.workloads` holds the named workloads and seeded inputs.
Importing the package does not load the library; the first call does, and raises if the
library is missing (there is no CPU fallback).
"""
