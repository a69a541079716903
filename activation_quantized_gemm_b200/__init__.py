"""B200-native symmetric INT8 activation-quantized GEMM (sm_100a CUDA behind a C ABI).

``activation_quantized_gemm_b200.i8q`` is the thin ctypes binding over
``libi8q.so``; ``activation_quantized_gemm_b200.synth`` makes seeded synthetic
inputs.  Importing the package loads nothing; the library is loaded on first
use and raises if it is missing or cannot reach a CUDA device.
"""
__all__ = ["i8q", "synth"]
