"""B200-native (sm_100a) DeepSeek Sparse Attention hot path.

The CUDA library (``libdsa_b200.so``, C ABI in ``include/dsa.h``) holds every
kernel; ``long_context_fp8_b200.dsa`` is its thin Python binding.  Importing
the package loads nothing; the first call through ``dsa`` loads the library
and raises if it was not built.
"""
__all__ = ["dsa", "build"]
