"""B200-native BitNet b1.58 BitLinear forward (sm_100a CUDA kernels behind a C ABI).

The compute path is libbitnet.so (include/bitnet.h).  ``bitlinear_bitnet_quant_b200.api``
is its thin Python binding (imports torch), ``workloads`` the seeded synthetic
inputs and ``build_lib`` the in-tree nvcc build.
"""
