"""B200-native W4 + per-token-gated low-rank Error Compensator linear layer.

The CUDA library (libspear_w4ec.so, C ABI in include/spear_w4ec.h) does all
the work; ``w4_gemm_error_b200.spear`` is its Python binding.  Importing the
binding raises if the library is missing, so no code path here can fall back
to a CPU implementation.
"""

__all__ = ["spear", "inputs", "build"]
