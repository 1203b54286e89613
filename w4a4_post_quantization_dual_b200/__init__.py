"""DualQuant dual-scale W4A4 linear for NVIDIA B200 (sm_100a).

The compute lives in the CUDA library libdq.so (C ABI, include/dq.h); the
Python binding in `dq` only marshals arguments.  Importing this package does
not load the library; the first call through `dq` does, and fails loudly if
it is missing.
"""
__all__ = ["dq", "synth"]
