"""B200-native (sm_100a) AWQ group-wise W4A16 library: quantise/pack, scale search,
fused dequantising GEMV and tcgen05 GEMM, behind the C ABI in include/awq.h.

Submodules: `awq` (the ctypes binding of the C ABI) and `build` (compiles the
in-tree shared library with nvcc for sm_100a).
"""
