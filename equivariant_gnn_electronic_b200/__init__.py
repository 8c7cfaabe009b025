"""B200-native eSCN (SO(2)-equivariant) edge layer for electronic-structure GNNs.

The compute lives in libegnn.so (hand-written sm_100a CUDA behind the C ABI of
include/egnn.h); ``egnn`` is its ctypes binding.  Import ``egnn`` explicitly:
importing this package alone does not load the library, so that the build
step can run before it exists.
"""
