"""B200-native ternary-weight decode path: packed ternary GEMV / GEMM kernels.

The CUDA library is loaded on first use of a binding function (``tern``);
importing this package does not touch the GPU.
"""
