"""B200 (sm_100a) implementation of the Native Sparse Attention per-layer operator.

The operator runs in libnsa.so (hand-written CUDA behind the C ABI of
include/nsa.h); ``nsa`` is its thin Python binding and ``inputs`` the seeded
synthetic input generator.  Import ``sparse_attention_long_phi_b200.nsa`` to
use the operator; it raises if the library is not built.
"""
