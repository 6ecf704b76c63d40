"""B200-native shared-negatives sampled-softmax cross-entropy LM head.

The compute lives in a C-ABI shared library of sm_100a CUDA kernels
(``libsampled_ce.so``, built in-tree); ``sampled_softmax_cross_b200.capi``
binds it with ctypes. Importing this package does not load the library; the
first call does, and fails loudly if it is missing.
"""
