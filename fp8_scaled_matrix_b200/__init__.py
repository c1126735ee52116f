"""FP8 (e4m3) scaled matrix multiply and dynamic quantizer for B200 (sm_100a).

The product is the C-ABI library libfp8sm.so (include/fp8sm.h); this package
holds its CUDA sources (csrc/), the build script, a ctypes binding with the
C names (fp8sm.py) and the seeded workload generators (workloads.py).
Import the binding explicitly: ``from fp8_scaled_matrix_b200 import fp8sm``.
"""
__all__ = ["fp8sm", "workloads", "build"]
