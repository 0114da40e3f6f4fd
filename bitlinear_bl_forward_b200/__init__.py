"""B200-native BitNet b1.58 BitLinear forward (sm_100a).

The compute lives in ``libbitlinear.so`` (hand-written CUDA kernels behind a
C ABI declared in ``include/bitlinear.h``).  ``bitlinear_bl_forward_b200.bl``
is the thin Python binding; importing this package does not load the library.
"""
