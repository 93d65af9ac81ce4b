"""B200-native low-rank (SVD-factorized) transformer inference hot path.

The compute path is the C-ABI library ``libflashsvd.so`` (CUDA kernels for
sm_100a); :mod:`rank_transformer_b200.flashsvd` is its ctypes binding and
:mod:`rank_transformer_b200.model` drives whole models through it.  Importing
this package does not load the library; importing ``flashsvd`` does, and fails
loudly if it is missing.
"""
